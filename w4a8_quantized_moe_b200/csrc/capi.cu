// capi.cu - the extern "C" entry points declared in include/w4a8.h: argument
// checks, workspace layout, TMA descriptors and the launch sequence.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <climits>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/w4a8.h"
#include "internal.h"

namespace w4a8 {
cudaError_t read_and_clear_device_error(int* value);
const char* set_last_error(const char* msg);
}

using namespace w4a8;

namespace {

thread_local std::string g_last_error;

w4a8_status fail(w4a8_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

w4a8_status cuda_fail(cudaError_t err, const char* where) {
  return fail(W4A8_ERR_CUDA, "%s: %s", where, cudaGetErrorString(err));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
  int major = 0;
  int sms = 0;
};

// Current device's compute capability and SM count (cached per device).
w4a8_status device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  DeviceInfo d;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && have[dev]) d = cache[dev];
  }
  if (d.sms == 0) {
    err = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return cuda_fail(err, "cudaDeviceGetAttribute");
    if (dev < 64) {
      std::lock_guard<std::mutex> lock(mu);
      cache[dev] = d;
      have[dev] = true;
    }
  }
  *out = d;
  if (d.major != 10)
    return fail(W4A8_ERR_UNSUPPORTED_ARCH,
                "device compute capability %d.x; this library is built for sm_100a (10.x)",
                d.major);
  return W4A8_OK;
}

// Bump allocator over the caller's workspace (or over nullptr to size it).
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~static_cast<size_t>(255);
    T* p = reinterpret_cast<T*>(base + off);
    off += count * sizeof(T);
    return p;
  }
};

struct RouteBufs {
  int32_t* block_counts;
  int32_t* block_base;
  int32_t* tile_prefix;
  int32_t* tile_prefix_wide;  // split tiling: the wide-tile table
};

RouteBufs carve_route(Carver& c, int64_t T, int E, bool wide_table = false) {
  RouteBufs b;
  const size_t n = static_cast<size_t>(route_blocks(T)) * static_cast<size_t>(E);
  b.block_counts = c.take<int32_t>(n);
  b.block_base = c.take<int32_t>(n);
  b.tile_prefix = c.take<int32_t>(static_cast<size_t>(E) + 1);
  b.tile_prefix_wide = wide_table ? c.take<int32_t>(static_cast<size_t>(E) + 1) : nullptr;
  return b;
}

struct ForwardBufs {
  int32_t* topk_ids;
  float* topk_w;
  int32_t* expert_offsets;
  int32_t* sorted_token_ids;
  int32_t* row_of;
  RouteBufs route;
  uint8_t* act_codes;
  uint8_t* perm_codes;
  float* act_scales;
  float* act_gsum;
  float* h;
  uint32_t* row_amax;
  uint8_t* inter_codes;
  float* inter_scales;
  float* inter_gsum;
  uint16_t* act_parts;    // [A, sum_parts_ld(H)] three-part bf16 group sums
  uint16_t* inter_parts;  // [A, sum_parts_ld(I)] the same for the intermediate codes
  int32_t* act_rowsum;    // INT8 variant: per token, sum of code + 128
  int32_t* inter_rowsum;  // INT8 variant: per segment row
  float* y;
};

ForwardBufs carve_forward(Carver& c, int64_t T, int64_t H, int64_t I, int E, int k) {
  ForwardBufs b;
  const size_t A = static_cast<size_t>(T) * static_cast<size_t>(k);
  b.topk_ids = c.take<int32_t>(A);
  b.topk_w = c.take<float>(A);
  b.expert_offsets = c.take<int32_t>(static_cast<size_t>(E) + 1);
  b.sorted_token_ids = c.take<int32_t>(A);
  b.row_of = c.take<int32_t>(A);
  b.route = carve_route(c, T, E, true);
  b.act_codes = c.take<uint8_t>(static_cast<size_t>(T) * static_cast<size_t>(H));
  b.perm_codes = c.take<uint8_t>(A * static_cast<size_t>(H));
  b.act_scales = c.take<float>(static_cast<size_t>(T));
  b.act_gsum = c.take<float>(static_cast<size_t>(T) * static_cast<size_t>(H / kGroup));
  b.h = c.take<float>(A * static_cast<size_t>(I));
  b.row_amax = c.take<uint32_t>(A);
  b.inter_codes = c.take<uint8_t>(A * static_cast<size_t>(I));
  b.inter_scales = c.take<float>(A);
  b.inter_gsum = c.take<float>(A * static_cast<size_t>(I / kGroup));
  b.act_parts = c.take<uint16_t>(A * static_cast<size_t>(sum_parts_ld(H)));
  b.inter_parts = c.take<uint16_t>(A * static_cast<size_t>(sum_parts_ld(I)));
  b.act_rowsum = c.take<int32_t>(static_cast<size_t>(T));
  b.inter_rowsum = c.take<int32_t>(A);
  b.y = c.take<float>(A * static_cast<size_t>(H));
  return b;
}

// The FP8-block shared expert's scratch.
struct SharedBufs {
  uint8_t* act_codes;   // [T, H] E4M3 codes, per-token-group scaled
  float* act_scales;    // [T, H / 128]
  float* h;             // [T, I] float32 SwiGLU output
  uint8_t* h_codes;     // [T, I]
  float* h_scales;      // [T, I / 128]
  int32_t* tables;      // [4]: expert offsets {0, T}, tile prefix {0, tiles}
  float* y;             // [T, H] float32 output (the combined layer only)
};

SharedBufs carve_shared(Carver& c, int64_t T, int64_t H, int64_t I, bool with_y) {
  SharedBufs b;
  const size_t t = static_cast<size_t>(T);
  b.act_codes = c.take<uint8_t>(t * static_cast<size_t>(H));
  b.act_scales = c.take<float>(t * static_cast<size_t>(H / kGroup));
  b.h = c.take<float>(t * static_cast<size_t>(I));
  b.h_codes = c.take<uint8_t>(t * static_cast<size_t>(I));
  b.h_scales = c.take<float>(t * static_cast<size_t>(I / kGroup));
  b.tables = c.take<int32_t>(4);
  b.y = with_y ? c.take<float>(t * static_cast<size_t>(H)) : nullptr;
  return b;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D byte tensor [outer, inner] with row pitch `inner` bytes.
w4a8_status encode_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                         uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(W4A8_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(W4A8_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for [%llu x %llu]",
                static_cast<int>(r), static_cast<unsigned long long>(outer),
                static_cast<unsigned long long>(inner));
  return W4A8_OK;
}

// Tile order within an expert: token blocks fastest for the wide (prefill)
// tiles, where several token blocks share each weight-row block;
// W4A8_TILE_ORDER = 0 / 1 forces weight-block-major / token-block-fastest.
int tile_order_nb_fastest(bool decode) {
  static const int forced = [] {
    const char* s = std::getenv("W4A8_TILE_ORDER");
    return s ? std::atoi(s) : -1;
  }();
  return forced >= 0 ? (forced != 0) : (decode ? 0 : 1);
}

// Average tokens per expert up to which w4a8_moe_forward uses the decode shape.
constexpr int kDecodeTokensPerExpert = 32;

// Split tiling: from this many assignments per expert on average, the experts
// with more than kTileNDecode segment rows run in the wide (prefill) tile
// shape and the rest in the narrow (decode) shape, as two launches of each
// grouped GEMM (a skewed batch has both kinds).  W4A8_SPLIT_TILES = 0 / 1
// turns it off / on for every batch.
constexpr int kSplitTokensPerExpert = 8;

bool split_tiles(int64_t A, int64_t E) {
  static const int forced = [] {
    const char* v = std::getenv("W4A8_SPLIT_TILES");
    return v ? std::atoi(v) : -1;
  }();
  // a forced shape that removes the offset once per tile needs per-row group
  // sums that only one regime's quantisers write: no split then
  if (grouped_gemm_uses_sum_parts(true) || grouped_gemm_uses_sum_parts(false)) return false;
  if (forced >= 0) return forced != 0;
  return A >= static_cast<int64_t>(kSplitTokensPerExpert) * E;
}

// Both launches of one grouped GEMM under split tiling: the narrow-tile
// (decode) shape over the experts with tiles in a.tile_prefix, then the
// wide-tile (prefill) shape over those in tile_prefix_wide.
cudaError_t launch_grouped_gemm_split(bool gate_up, const CUtensorMap& tw, const CUtensorMap& ta,
                                      const CUtensorMap& tsc, const CUtensorMap& tgs,
                                      const GemmArgs& a, const int32_t* tile_prefix_wide,
                                      int num_sms, cudaStream_t s) {
  cudaError_t err = launch_grouped_gemm(gate_up, true, tw, ta, tsc, tgs, a, num_sms, s);
  if (err != cudaSuccess) return err;
  GemmArgs w = a;
  w.tile_prefix = tile_prefix_wide;
  w.nb_fastest = tile_order_nb_fastest(false);
  return launch_grouped_gemm(gate_up, false, tw, ta, tsc, tgs, w, num_sms, s);
}

uint64_t wait_timeout_ns() {
  static uint64_t v = [] {
    const char* s = std::getenv("W4A8_WAIT_TIMEOUT_MS");
    uint64_t ms = s ? std::strtoull(s, nullptr, 10) : 0;
    if (ms == 0) ms = 2000;
    return ms * 1000000ull;
  }();
  return v;
}

w4a8_status check_route_args(const void* logits, int64_t T, int32_t E, int32_t k) {
  if (T < 0) return fail(W4A8_ERR_INVALID_ARG, "T = %lld < 0", static_cast<long long>(T));
  if (E < 1 || E > kMaxExperts)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "E = %d outside [1, %d]", E, kMaxExperts);
  if (k < 1 || k > E || k > kMaxTopK)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "k = %d outside [1, min(E, %d)]", k, kMaxTopK);
  if (T * static_cast<int64_t>(k) > INT32_MAX)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "T * k exceeds 2^31 - 1");
  if (T > 0 && !logits) return fail(W4A8_ERR_INVALID_ARG, "logits is NULL");
  if (!aligned16(logits)) return fail(W4A8_ERR_INVALID_ARG, "logits is not 16-byte aligned");
  return W4A8_OK;
}

}  // namespace

namespace w4a8 {
// Records the message w4a8_last_error() returns on this thread.
const char* set_last_error(const char* msg) {
  g_last_error = msg;
  return g_last_error.c_str();
}
}  // namespace w4a8

namespace {
w4a8_status pack_int4_common(const char* name, const void* w_bf16, int64_t R, int64_t K,
                             int32_t group, int32_t* packed, void* scales_bf16, bool clip,
                             void* stream) {
  if (group != kGroup) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "group = %d; only 128", group);
  if (R < 0 || K <= 0) return fail(W4A8_ERR_INVALID_ARG, "R = %lld, K = %lld",
                                   static_cast<long long>(R), static_cast<long long>(K));
  if (K % kGroup) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "K = %lld is not a multiple of 128",
                              static_cast<long long>(K));
  if (R == 0) return W4A8_OK;
  if (!w_bf16 || !packed || !scales_bf16) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(w_bf16) || !aligned16(packed) || !aligned16(scales_bf16))
    return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_pack_int4(w_bf16, R, K, packed, scales_bf16, clip, di.sms,
                                     static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, name);
}
}  // namespace

extern "C" {

int32_t w4a8_abi_version(void) { return 1; }

int32_t w4a8_build_flags(void) {
#if W4A8_DEBUG_BOUNDS
  return W4A8_BUILD_DEBUG_BOUNDS;
#else
  return 0;
#endif
}

const char* w4a8_status_string(w4a8_status s) {
  switch (s) {
    case W4A8_OK: return "W4A8_OK";
    case W4A8_ERR_INVALID_ARG: return "W4A8_ERR_INVALID_ARG";
    case W4A8_ERR_UNSUPPORTED_SHAPE: return "W4A8_ERR_UNSUPPORTED_SHAPE";
    case W4A8_ERR_UNSUPPORTED_ARCH: return "W4A8_ERR_UNSUPPORTED_ARCH";
    case W4A8_ERR_WORKSPACE_TOO_SMALL: return "W4A8_ERR_WORKSPACE_TOO_SMALL";
    case W4A8_ERR_CUDA: return "W4A8_ERR_CUDA";
    case W4A8_ERR_DEVICE_TIMEOUT: return "W4A8_ERR_DEVICE_TIMEOUT";
    case W4A8_ERR_DEVICE_INDEX: return "W4A8_ERR_DEVICE_INDEX";
    default: return "W4A8_ERR_UNKNOWN";
  }
}

const char* w4a8_last_error(void) { return g_last_error.c_str(); }

w4a8_status w4a8_check_device_error(void* stream) {
  cudaError_t err = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "cudaStreamSynchronize");
  int v = 0;
  err = read_and_clear_device_error(&v);
  if (err != cudaSuccess) return cuda_fail(err, "reading the device error latch");
  if (v & kDeviceErrorTimeout)
    return fail(W4A8_ERR_DEVICE_TIMEOUT, "a bounded in-kernel wait ran out (latch 0x%x)", v);
  if (v & kDeviceErrorIndex)
    return fail(W4A8_ERR_DEVICE_INDEX,
                "an index read on the device was out of range; the access was skipped (latch 0x%x)",
                v);
  return W4A8_OK;
}

w4a8_status w4a8_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull)
    return fail(W4A8_ERR_INVALID_ARG, "timeout_ns = %llu; need 0 < timeout_ns <= 10 s",
                static_cast<unsigned long long>(timeout_ns));
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_wait_timeout_selftest(timeout_ns, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "self-test launch");
}

w4a8_status w4a8_pack_int4(const void* w_bf16, int64_t R, int64_t K, int32_t group,
                           int32_t* packed, void* scales_bf16, void* stream) {
  return pack_int4_common("pack_int4 launch", w_bf16, R, K, group, packed, scales_bf16, false,
                          stream);
}

w4a8_status w4a8_pack_int4_mse_clip(const void* w_bf16, int64_t R, int64_t K, int32_t group,
                                    int32_t* packed, void* scales_bf16, void* stream) {
  return pack_int4_common("pack_int4_mse_clip launch", w_bf16, R, K, group, packed, scales_bf16,
                          true, stream);
}

w4a8_status w4a8_quant_act_fp8_per_token(const void* x_bf16, int64_t T, int64_t H,
                                         uint8_t* codes_e4m3, float* scales, void* stream) {
  if (T < 0 || H <= 0) return fail(W4A8_ERR_INVALID_ARG, "T = %lld, H = %lld",
                                   static_cast<long long>(T), static_cast<long long>(H));
  if (H % 16) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "H = %lld is not a multiple of 16",
                          static_cast<long long>(H));
  if (T == 0) return W4A8_OK;
  if (!x_bf16 || !codes_e4m3 || !scales) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(x_bf16) || !aligned16(codes_e4m3) || !aligned16(scales))
    return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_act_quant(x_bf16, T, H, codes_e4m3, scales, nullptr, nullptr, 0, nullptr, di.sms,
                                     static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "act_quant launch");
}

w4a8_status w4a8_prepare_experts_b200(const int32_t* packed, const void* scales_bf16, int64_t E,
                                      int64_t rows, int64_t K, int32_t* packed_out,
                                      void* scales_out, void* stream) {
  if (E < 0 || rows < 0 || K <= 0)
    return fail(W4A8_ERR_INVALID_ARG, "E = %lld, rows = %lld, K = %lld", static_cast<long long>(E),
                static_cast<long long>(rows), static_cast<long long>(K));
  if (K % kGroup) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "K = %lld is not a multiple of 128",
                              static_cast<long long>(K));
  const int64_t nwords = E * rows * (K / 8);
  const int64_t nscales = E * rows * (K / kGroup);
  if (nwords == 0) return W4A8_OK;
  if (!packed || !scales_bf16 || !packed_out || !scales_out)
    return fail(W4A8_ERR_INVALID_ARG, "NULL pointer");
  for (const void* p : {static_cast<const void*>(packed), scales_bf16,
                        static_cast<const void*>(packed_out), static_cast<const void*>(scales_out)})
    if (!aligned16(p)) return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (packed != packed_out && packed < packed_out + nwords && packed_out < packed + nwords)
    return fail(W4A8_ERR_INVALID_ARG, "packed and packed_out overlap without being the same buffer");
  const uint8_t* si = static_cast<const uint8_t*>(scales_bf16);
  const uint8_t* so = static_cast<const uint8_t*>(scales_out);
  if (si < so + 2 * nscales && so < si + 2 * nscales)
    return fail(W4A8_ERR_INVALID_ARG, "scales and scales_out overlap");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = launch_repack_int4_b200(packed, nwords, packed_out, di.sms, s);
  if (err == cudaSuccess)
    err = launch_transpose_scales(scales_bf16, E, rows, K / kGroup, scales_out, di.sms, s);
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "prepare_experts launch");
}

size_t w4a8_moe_route_workspace_size(int64_t T, int32_t E) {
  if (T < 0 || E < 1) return 0;
  Carver c(nullptr);
  carve_route(c, T, E);
  return c.off + 256;
}

w4a8_status w4a8_moe_route_permute(const float* logits, int64_t T, int32_t E, int32_t k,
                                   int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                                   int32_t* sorted_token_ids, int32_t* row_of, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (w4a8_status st = check_route_args(logits, T, E, k)) return st;
  if (!expert_offsets || !workspace)
    return fail(W4A8_ERR_INVALID_ARG, "expert_offsets / workspace is NULL");
  if (T > 0 && (!topk_ids || !topk_w || !sorted_token_ids || !row_of))
    return fail(W4A8_ERR_INVALID_ARG, "NULL output pointer");
  for (const void* p : {static_cast<const void*>(topk_ids), static_cast<const void*>(topk_w),
                        static_cast<const void*>(expert_offsets),
                        static_cast<const void*>(sorted_token_ids),
                        static_cast<const void*>(row_of), static_cast<const void*>(workspace)})
    if (!aligned16(p)) return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = w4a8_moe_route_workspace_size(T, E);
  if (workspace_bytes < need)
    return fail(W4A8_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu", workspace_bytes, need);
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  Carver c(workspace);
  RouteBufs rb = carve_route(c, T, E);
  cudaError_t err = launch_route(logits, T, E, k, topk_ids, topk_w, expert_offsets,
                                 sorted_token_ids, row_of, rb.block_counts, rb.block_base,
                                 rb.tile_prefix, kTileNPrefill, nullptr,
                                 static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "route launch");
}

int32_t w4a8_moe_forward_launches(int64_t T, int32_t E, int32_t k) {
  if (T <= 0 || E < 1 || k < 1) return 0;
  // activation quantiser, top-k, scan, scatter, two grouped GEMMs, the
  // requantiser and the combine; split tiling launches each GEMM twice
  return split_tiles(T * k, E) ? 10 : 8;
}

size_t w4a8_moe_workspace_size(int64_t T, int64_t H, int64_t I, int32_t E, int32_t k) {
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return 0;
  Carver c(nullptr);
  carve_forward(c, T, H, I, E, k);
  return c.off + 256;
}

}  // extern "C"

namespace {
w4a8_status check_shared_shape(int64_t T, int64_t H, int64_t I) {
  if (T < 0) return fail(W4A8_ERR_INVALID_ARG, "T = %lld < 0", static_cast<long long>(T));
  if (H <= 0 || I <= 0 || H % kGroup || I % kGroup)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE,
                "shared expert: H = %lld and I = %lld must be positive multiples of 128",
                static_cast<long long>(H), static_cast<long long>(I));
  if (H / kGroup > kMaxGroups || I / kGroup > kMaxGroups)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "shared expert: at most %d groups of 128 per row",
                kMaxGroups);
  if (T > INT32_MAX) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "T exceeds 2^31 - 1");
  return W4A8_OK;
}

// The FP8-block shared expert for T rows of hidden: group-quantise x, gate/up
// GEMM + SwiGLU, group-requantise h, down GEMM into y [T, H] float32.
// Stage events (aux->stage_events, 8 handles): 0/1 input quantisation, 2/3
// gate/up GEMM, 4/5 requantisation of h, 6/7 down GEMM.
// The FP8-block shared expert's steps, set up once per call: its tensor maps,
// GEMM arguments and stage events.  The steps run in order; in a routed
// decode call its two GEMMs run inside the routed GEMM launches instead.
struct SharedRun {
  CUtensorMap tw1, ta1, tw2, ta2;
  GemmArgs g1, g2;
  int ctas1 = 0, ctas2 = 0, tile_n = 0;
  SharedBufs b;
  const void* hidden = nullptr;
  int64_t T = 0, H = 0, I = 0;
  void* const* ev = nullptr;
};

cudaError_t shared_record(const SharedRun& r, int i, cudaStream_t s) {
  return r.ev && r.ev[i] ? cudaEventRecord(static_cast<cudaEvent_t>(r.ev[i]), s) : cudaSuccess;
}

// tile_n: token rows per tile of the shared expert's GEMM shape
w4a8_status shared_setup(SharedRun& r, const void* hidden_bf16, const uint8_t* w13_codes,
                         const float* w13_scales, const uint8_t* w2_codes,
                         const float* w2_scales, int64_t T, int64_t H, int64_t I, float* y,
                         SharedBufs b, const w4a8_shared_aux* aux, const DeviceInfo& di,
                         int tile_n) {
  if (aux) {
    auto pick = [](auto* user, auto* ws) { return user ? user : ws; };
    b.act_codes = pick(aux->act_codes, b.act_codes);
    b.act_scales = pick(aux->act_scales, b.act_scales);
    b.h = pick(aux->h, b.h);
    b.h_codes = pick(aux->h_codes, b.h_codes);
    b.h_scales = pick(aux->h_scales, b.h_scales);
    for (const void* p : {static_cast<const void*>(b.act_codes), static_cast<const void*>(b.act_scales),
                          static_cast<const void*>(b.h), static_cast<const void*>(b.h_codes),
                          static_cast<const void*>(b.h_scales)})
      if (!aligned16(p)) return fail(W4A8_ERR_INVALID_ARG, "aux buffers must be 16-byte aligned");
    r.ev = aux->stage_events;
  }
  r.b = b;
  r.hidden = hidden_bf16;
  r.T = T;
  r.H = H;
  r.I = I;
  r.tile_n = tile_n;
  // E4M3 weights [rows, K] bytes, 128-byte swizzle: boxes of 64 rows (the
  // gate and up halves of a gate/up tile) or 128 rows (down); activation codes
  // [T, K] in 16-row boxes, as for the routed experts.
  if (w4a8_status st = encode_u8_2d(&r.tw1, w13_codes, static_cast<uint64_t>(H),
                                    static_cast<uint64_t>(2 * I), 128, 64,
                                    CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&r.ta1, b.act_codes, static_cast<uint64_t>(H),
                                    static_cast<uint64_t>(T), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&r.tw2, w2_codes, static_cast<uint64_t>(I),
                                    static_cast<uint64_t>(H), 128, 128,
                                    CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&r.ta2, b.h_codes, static_cast<uint64_t>(I),
                                    static_cast<uint64_t>(T), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  const int64_t tiles_n = (T + tile_n - 1) / tile_n;
  GemmArgs& g1 = r.g1;
  g1 = GemmArgs{};
  g1.K = static_cast<int>(H);
  g1.n_rows = static_cast<int>(2 * I);
  g1.half_rows = static_cast<int>(I);
  g1.E = 1;
  g1.expert_offsets = b.tables;
  g1.tile_prefix = b.tables + 2;
  g1.act_gsum = b.act_scales;
  g1.wscale = w13_scales;
  g1.out = b.h;
  g1.out_ld = I;
  g1.act_rows = T;
  g1.timeout_ns = wait_timeout_ns();
  g1.nb_fastest = 1;
  g1.n_seg_rows = T;
  g1.n_tokens = T;
  r.ctas1 = static_cast<int>(std::min<int64_t>(tiles_n * (I / 64), di.sms));
  GemmArgs& g2 = r.g2;
  g2 = g1;
  g2.K = static_cast<int>(I);
  g2.n_rows = static_cast<int>(H);
  g2.half_rows = 0;
  g2.act_gsum = b.h_scales;
  g2.wscale = w2_scales;
  g2.out = y;
  g2.out_ld = H;
  r.ctas2 = static_cast<int>(std::min<int64_t>(tiles_n * (H / kGroup), di.sms));
  return W4A8_OK;
}

#define W4A8_STEP(call, what)                              \
  do {                                                     \
    cudaError_t err_ = (call);                             \
    if (err_ != cudaSuccess) return cuda_fail(err_, what); \
  } while (0)

// the dense tables of the one expert, and the input's group quantisation
w4a8_status shared_front(const SharedRun& r, const DeviceInfo& di, cudaStream_t s) {
  W4A8_STEP(launch_dense_tables(r.b.tables, r.b.tables + 2, r.T, r.tile_n, s),
            "dense tables launch");
  W4A8_STEP(shared_record(r, 0, s), "cudaEventRecord");
  W4A8_STEP(launch_act_quant_group(r.hidden, nullptr, r.T, r.H, r.b.act_codes, r.b.act_scales,
                                   di.sms, s),
            "shared input quantisation launch");
  W4A8_STEP(shared_record(r, 1, s), "cudaEventRecord");
  return W4A8_OK;
}

w4a8_status shared_gemm(const SharedRun& r, bool gate_up, cudaStream_t s) {
  W4A8_STEP(shared_record(r, gate_up ? 2 : 6, s), "cudaEventRecord");
  W4A8_STEP(gate_up ? launch_fp8_block_gemm(true, r.tw1, r.ta1, r.g1, r.ctas1, s)
                    : launch_fp8_block_gemm(false, r.tw2, r.ta2, r.g2, r.ctas2, s),
            gate_up ? "shared gate/up GEMM launch" : "shared down GEMM launch");
  W4A8_STEP(shared_record(r, gate_up ? 3 : 7, s), "cudaEventRecord");
  return W4A8_OK;
}

// h requantised per token and 128-group
w4a8_status shared_mid(const SharedRun& r, const DeviceInfo& di, cudaStream_t s) {
  W4A8_STEP(shared_record(r, 4, s), "cudaEventRecord");
  W4A8_STEP(launch_act_quant_group(nullptr, r.b.h, r.T, r.I, r.b.h_codes, r.b.h_scales, di.sms,
                                   s),
            "shared intermediate quantisation launch");
  W4A8_STEP(shared_record(r, 5, s), "cudaEventRecord");
  return W4A8_OK;
}
#undef W4A8_STEP

w4a8_status shared_forward_impl(const void* hidden_bf16, const uint8_t* w13_codes,
                                const float* w13_scales, const uint8_t* w2_codes,
                                const float* w2_scales, int64_t T, int64_t H, int64_t I,
                                float* y, SharedBufs b, const w4a8_shared_aux* aux,
                                const DeviceInfo& di, cudaStream_t s) {
  SharedRun r;
  if (w4a8_status st = shared_setup(r, hidden_bf16, w13_codes, w13_scales, w2_codes, w2_scales, T,
                                    H, I, y, b, aux, di, grouped_gemm_tile_n(false)))
    return st;
  if (w4a8_status st = shared_front(r, di, s)) return st;
  if (w4a8_status st = shared_gemm(r, true, s)) return st;
  if (w4a8_status st = shared_mid(r, di, s)) return st;
  return shared_gemm(r, false, s);
}

// Whether a routed decode call runs the shared expert's GEMMs inside its own
// GEMM launches (W4A8_SHARED_FUSED = 0 keeps them apart).
bool shared_fused_by_default() {
  static const int v = [] {
    const char* e = std::getenv("W4A8_SHARED_FUSED");
    return e ? std::atoi(e) : 1;
  }();
  return v != 0;
}

// The layer's optional FP8-block shared expert.
struct SharedExpert {
  const uint8_t* w13_codes;
  const float* w13_scales;
  const uint8_t* w2_codes;
  const float* w2_scales;
  int64_t I;
  const w4a8_shared_aux* aux;
};

// The layer, for both variants: i8 == nullptr runs the W4A8 (FP8 E4M3
// activations, group-128 scales) path; otherwise the per-channel INT4 x
// per-token INT8 path with i8 = {w13 nibble row sums, w2 nibble row sums}.
struct Int8Weights {
  const int32_t* w13_nsum;
  const int32_t* w2_nsum;
};

w4a8_status moe_forward_impl(const void* hidden_bf16, const float* logits,
                             const int32_t* w13_packed, const void* w13_scales,
                             const int32_t* w2_packed, const void* w2_scales, int64_t T,
                             int64_t H, int64_t I, int32_t E, int32_t k, void* out_bf16,
                             void* workspace, size_t workspace_bytes, const w4a8_moe_aux* aux,
                             void* stream, const Int8Weights* i8,
                             const SharedExpert* sh = nullptr) {
  if (w4a8_status st = check_route_args(logits, T, E, k)) return st;
  if (sh) {
    if (w4a8_status st = check_shared_shape(T, H, sh->I)) return st;
    const void* sp[] = {sh->w13_codes, sh->w13_scales, sh->w2_codes, sh->w2_scales};
    for (const void* p : sp)
      if (T > 0 && (!p || !aligned16(p)))
        return fail(W4A8_ERR_INVALID_ARG, "shared expert pointers must be non-NULL and 16-byte aligned");
  }
  if (H <= 0 || I <= 0 || H % kGroup || I % kGroup)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "H = %lld and I = %lld must be positive multiples of 128",
                static_cast<long long>(H), static_cast<long long>(I));
  if (H / kGroup > kMaxGroups || I / kGroup > kMaxGroups)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "H = %lld, I = %lld: at most %d groups of 128 per row",
                static_cast<long long>(H), static_cast<long long>(I), kMaxGroups);
  if (static_cast<int64_t>(E) * 2 * I > INT32_MAX || static_cast<int64_t>(E) * H > INT32_MAX)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "E * rows exceeds 2^31 - 1");
  if (T == 0) return W4A8_OK;
  const void* ptrs[] = {hidden_bf16, w13_packed, w13_scales, w2_packed, w2_scales, out_bf16,
                        workspace, i8 ? i8->w13_nsum : workspace, i8 ? i8->w2_nsum : workspace};
  for (const void* p : ptrs) {
    if (!p) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(p)) return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  const size_t need = sh ? w4a8_moe_shared_workspace_size(T, H, I, E, k, sh->I)
                         : w4a8_moe_workspace_size(T, H, I, E, k);
  if (workspace_bytes < need)
    return fail(W4A8_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu", workspace_bytes, need);
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  Carver c(workspace);
  ForwardBufs b = carve_forward(c, T, H, I, E, k);
  SharedBufs sb{};
  if (sh) sb = carve_shared(c, T, H, sh->I, true);
  void* const* ev = nullptr;
  if (aux) {
    auto pick = [](auto* user, auto* ws) { return user ? user : ws; };
    b.topk_ids = pick(aux->topk_ids, b.topk_ids);
    b.topk_w = pick(aux->topk_w, b.topk_w);
    b.expert_offsets = pick(aux->expert_offsets, b.expert_offsets);
    b.sorted_token_ids = pick(aux->sorted_token_ids, b.sorted_token_ids);
    b.row_of = pick(aux->row_of, b.row_of);
    b.act_codes = pick(aux->act_codes, b.act_codes);
    b.act_scales = pick(aux->act_scales, b.act_scales);
    b.h = pick(aux->inter_h, b.h);
    b.inter_codes = pick(aux->inter_codes, b.inter_codes);
    b.inter_scales = pick(aux->inter_scales, b.inter_scales);
    b.y = pick(aux->y_rows, b.y);
    for (const void* p : {static_cast<const void*>(b.topk_ids), static_cast<const void*>(b.topk_w),
                          static_cast<const void*>(b.expert_offsets),
                          static_cast<const void*>(b.sorted_token_ids),
                          static_cast<const void*>(b.row_of), static_cast<const void*>(b.act_codes),
                          static_cast<const void*>(b.act_scales), static_cast<const void*>(b.h),
                          static_cast<const void*>(b.inter_codes),
                          static_cast<const void*>(b.inter_scales), static_cast<const void*>(b.y)})
      if (!aligned16(p)) return fail(W4A8_ERR_INVALID_ARG, "aux buffers must be 16-byte aligned");
    ev = aux->stage_events;
  }
  const int64_t A = T * k;
  // Few tokens per expert (decode): narrow tiles with a deep pipeline; many
  // (prefill): wide tiles that feed each converted weight tile to more tokens;
  // in between (split): each expert by its own count.
  const bool decode = A <= static_cast<int64_t>(kDecodeTokensPerExpert) * E;
  const bool split = !i8 && split_tiles(A, E);
  const int tile_n = split ? kTileNDecode : grouped_gemm_tile_n(decode);
  SplitTiles st;
  if (split) {
    st.wide_min = kTileNDecode;
    st.tile_n_wide = kTileNPrefill;
    st.tile_prefix_wide = b.route.tile_prefix_wide;
  }

  // TMA descriptors: packed weights [E * rows, K / 2] bytes, 64-byte swizzle;
  // activation codes in segment order [A, K] bytes, 128-byte swizzle, 16-row boxes.
  CUtensorMap tw1, ta1, tw2, ta2, ts1, ts2, tg1, tg2;
  if (w4a8_status st = encode_u8_2d(&tw1, w13_packed, static_cast<uint64_t>(H / 2),
                                    static_cast<uint64_t>(E) * 2 * I, 64, 64,
                                    CU_TENSOR_MAP_SWIZZLE_64B))
    return st;
  if (w4a8_status st = encode_u8_2d(&ta1, b.perm_codes, static_cast<uint64_t>(H),
                                    static_cast<uint64_t>(A), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&tw2, w2_packed, static_cast<uint64_t>(I / 2),
                                    static_cast<uint64_t>(E) * H, 64, 128,
                                    CU_TENSOR_MAP_SWIZZLE_64B))
    return st;
  if (w4a8_status st = encode_u8_2d(&ta2, b.inter_codes, static_cast<uint64_t>(I),
                                    static_cast<uint64_t>(A), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  // three-part group sums as bytes [A, 2 ld], 16 rows x 128 bytes per box
  const bool parts = !i8 && !split && grouped_gemm_uses_sum_parts(decode);
  if (w4a8_status st = encode_u8_2d(&tg1, b.act_parts, static_cast<uint64_t>(2 * sum_parts_ld(H)),
                                    static_cast<uint64_t>(A), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&tg2, b.inter_parts,
                                    static_cast<uint64_t>(2 * sum_parts_ld(I)),
                                    static_cast<uint64_t>(A), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  // group-major scales as bytes: [E * G, 2 * rows]; one box = one tile's scales
  // (W4A8 only; the INT8 variant reads its per-row scales in the epilogue)
  if (!i8) {
    if (w4a8_status st = encode_u8_2d(&ts1, w13_scales, static_cast<uint64_t>(2 * I) * 2,
                                      static_cast<uint64_t>(E) * (H / kGroup), 128,
                                      static_cast<uint32_t>(H / kGroup),
                                      CU_TENSOR_MAP_SWIZZLE_NONE))
      return st;
    if (w4a8_status st = encode_u8_2d(&ts2, w2_scales, static_cast<uint64_t>(H) * 2,
                                      static_cast<uint64_t>(E) * (I / kGroup), 256,
                                      static_cast<uint32_t>(I / kGroup),
                                      CU_TENSOR_MAP_SWIZZLE_NONE))
      return st;
  }

  auto record = [&](int i) -> cudaError_t {
    return ev && ev[i] ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) : cudaSuccess;
  };
  cudaError_t err = cudaSuccess;
#define W4A8_STEP(call, what)                     \
  do {                                            \
    err = (call);                                 \
    if (err != cudaSuccess) return cuda_fail(err, what); \
  } while (0)

  // the shared expert first: it reads only the hidden states, and the combine
  // adds its output
  // decode: the shared expert's two GEMMs run inside the routed GEMM launches
  // (their second phase, on the CTAs that finish their routed tiles first);
  // otherwise it runs first, in launches of its own
  const bool fuse_shared = sh && !i8 && !split && decode && shared_fused_by_default() &&
                           grouped_gemm_shared_fusable();
  SharedRun sr;
  if (sh) {
    if (w4a8_status st = shared_setup(sr, hidden_bf16, sh->w13_codes, sh->w13_scales,
                                      sh->w2_codes, sh->w2_scales, T, H, sh->I, sb.y, sb, sh->aux,
                                      di, fuse_shared ? grouped_gemm_shared_tile_n()
                                                      : grouped_gemm_tile_n(false)))
      return st;
    if (w4a8_status st = shared_front(sr, di, s)) return st;
    if (!fuse_shared) {
      if (w4a8_status st = shared_gemm(sr, true, s)) return st;
      if (w4a8_status st = shared_mid(sr, di, s)) return st;
      if (w4a8_status st = shared_gemm(sr, false, s)) return st;
    }
  }
  // routing first: the activation quantiser writes each token's codes to its
  // segment rows as well, so both GEMMs read contiguous activation tiles
  W4A8_STEP(record(2), "cudaEventRecord");
  W4A8_STEP(launch_route(logits, T, E, k, b.topk_ids, b.topk_w, b.expert_offsets,
                         b.sorted_token_ids, b.row_of, b.route.block_counts, b.route.block_base,
                         b.route.tile_prefix, tile_n, b.row_amax, s, st),
            "route launch");
  W4A8_STEP(record(3), "cudaEventRecord");
  W4A8_STEP(record(0), "cudaEventRecord");
  W4A8_STEP(launch_act_quant(hidden_bf16, T, H, b.act_codes, b.act_scales,
                             parts ? nullptr : b.act_gsum, b.row_of, k, b.perm_codes, di.sms, s,
                             i8 ? b.act_rowsum : nullptr, parts ? b.act_parts : nullptr),
            "act_quant launch");
  W4A8_STEP(record(1), "cudaEventRecord");

  GemmArgs g1{};
  g1.K = static_cast<int>(H);
  g1.n_rows = static_cast<int>(2 * I);
  g1.half_rows = static_cast<int>(I);
  g1.E = E;
  g1.expert_offsets = b.expert_offsets;
  g1.tile_prefix = b.route.tile_prefix;
  g1.row_tokens = b.sorted_token_ids;
  g1.act_scale = b.act_scales;
  g1.act_gsum = b.act_gsum;
  g1.wscale = w13_scales;
  g1.out = b.h;
  g1.out_ld = I;
  g1.row_amax = b.row_amax;
  g1.act_rows = T;
  g1.timeout_ns = wait_timeout_ns();
  g1.nb_fastest = tile_order_nb_fastest(decode);
  g1.n_seg_rows = A;
  g1.n_tokens = T;
  g1.wsum = i8 ? i8->w13_nsum : nullptr;
  g1.act_sum = b.act_rowsum;
  W4A8_STEP(record(4), "cudaEventRecord");
  if (split) {
    g1.nb_fastest = tile_order_nb_fastest(true);
    W4A8_STEP(launch_grouped_gemm_split(true, tw1, ta1, ts1, tg1, g1, b.route.tile_prefix_wide,
                                        di.sms, s),
              "gate/up GEMM launch");
  } else if (fuse_shared) {
    // the shared expert's gate/up stage events bracket nothing: its GEMM is
    // inside this launch
    W4A8_STEP(shared_record(sr, 2, s), "cudaEventRecord");
    W4A8_STEP(shared_record(sr, 3, s), "cudaEventRecord");
    W4A8_STEP(launch_grouped_gemm_with_shared(true, decode, tw1, ta1, ts1, tg1, sr.tw1, sr.ta1,
                                              g1, sr.g1, di.sms, s),
              "gate/up GEMM launch (with the shared expert)");
  } else {
    W4A8_STEP(i8 ? launch_grouped_gemm_i8(true, decode, tw1, ta1, g1, di.sms, s)
                 : launch_grouped_gemm(true, decode, tw1, ta1, ts1, tg1, g1, di.sms, s),
              "gate/up GEMM launch");
  }
  W4A8_STEP(record(5), "cudaEventRecord");

  W4A8_STEP(record(6), "cudaEventRecord");
  W4A8_STEP(launch_inter_quant(b.h, b.row_amax, A, I, b.inter_codes, b.inter_scales,
                               parts ? nullptr : b.inter_gsum, di.sms, s,
                               i8 ? b.inter_rowsum : nullptr, parts ? b.inter_parts : nullptr),
            "intermediate quant launch");
  W4A8_STEP(record(7), "cudaEventRecord");
  if (fuse_shared)
    if (w4a8_status st = shared_mid(sr, di, s)) return st;

  GemmArgs g2{};
  g2.K = static_cast<int>(I);
  g2.n_rows = static_cast<int>(H);
  g2.half_rows = 0;
  g2.E = E;
  g2.expert_offsets = b.expert_offsets;
  g2.tile_prefix = b.route.tile_prefix;
  g2.row_tokens = nullptr;
  g2.act_scale = b.inter_scales;
  g2.act_gsum = b.inter_gsum;
  g2.wscale = w2_scales;
  g2.out = b.y;
  g2.out_ld = H;
  g2.row_amax = nullptr;
  g2.act_rows = A;
  g2.timeout_ns = wait_timeout_ns();
  g2.nb_fastest = tile_order_nb_fastest(decode);
  g2.n_seg_rows = A;
  g2.n_tokens = T;
  g2.wsum = i8 ? i8->w2_nsum : nullptr;
  g2.act_sum = b.inter_rowsum;
  W4A8_STEP(record(8), "cudaEventRecord");
  if (split) {
    g2.nb_fastest = tile_order_nb_fastest(true);
    W4A8_STEP(launch_grouped_gemm_split(false, tw2, ta2, ts2, tg2, g2, b.route.tile_prefix_wide,
                                        di.sms, s),
              "down GEMM launch");
  } else if (fuse_shared) {
    W4A8_STEP(shared_record(sr, 6, s), "cudaEventRecord");
    W4A8_STEP(shared_record(sr, 7, s), "cudaEventRecord");
    W4A8_STEP(launch_grouped_gemm_with_shared(false, decode, tw2, ta2, ts2, tg2, sr.tw2, sr.ta2,
                                              g2, sr.g2, di.sms, s),
              "down GEMM launch (with the shared expert)");
  } else {
    W4A8_STEP(i8 ? launch_grouped_gemm_i8(false, decode, tw2, ta2, g2, di.sms, s)
                 : launch_grouped_gemm(false, decode, tw2, ta2, ts2, tg2, g2, di.sms, s),
              "down GEMM launch");
  }
  W4A8_STEP(record(9), "cudaEventRecord");

  W4A8_STEP(record(10), "cudaEventRecord");
  W4A8_STEP(launch_combine(b.y, b.row_of, b.topk_w, T, H, k, out_bf16, di.sms, s,
                           sh ? sb.y : nullptr),
            "combine launch");
  W4A8_STEP(record(11), "cudaEventRecord");
#undef W4A8_STEP
  return W4A8_OK;
}
}  // namespace

extern "C" {

w4a8_status w4a8_moe_forward(const void* hidden_bf16, const float* logits,
                             const int32_t* w13_packed, const void* w13_scales,
                             const int32_t* w2_packed, const void* w2_scales, int64_t T,
                             int64_t H, int64_t I, int32_t E, int32_t k, void* out_bf16,
                             void* workspace, size_t workspace_bytes, const w4a8_moe_aux* aux,
                             void* stream) {
  return moe_forward_impl(hidden_bf16, logits, w13_packed, w13_scales, w2_packed, w2_scales, T, H,
                          I, E, k, out_bf16, workspace, workspace_bytes, aux, stream, nullptr);
}

w4a8_status w4a8_moe_forward_channel_int8(const void* hidden_bf16, const float* logits,
                                          const int32_t* w13_packed, const void* w13_scales,
                                          const int32_t* w13_nibble_sums,
                                          const int32_t* w2_packed, const void* w2_scales,
                                          const int32_t* w2_nibble_sums, int64_t T, int64_t H,
                                          int64_t I, int32_t E, int32_t k, void* out_bf16,
                                          void* workspace, size_t workspace_bytes,
                                          const w4a8_moe_aux* aux, void* stream) {
  const Int8Weights i8{w13_nibble_sums, w2_nibble_sums};
  return moe_forward_impl(hidden_bf16, logits, w13_packed, w13_scales, w2_packed, w2_scales, T, H,
                          I, E, k, out_bf16, workspace, workspace_bytes, aux, stream, &i8);
}

w4a8_status w4a8_pack_int4_channel(const void* w_bf16, int64_t R, int64_t K, int32_t* packed,
                                   void* scales_bf16, void* stream) {
  if (R < 0 || K <= 0) return fail(W4A8_ERR_INVALID_ARG, "R = %lld, K = %lld",
                                   static_cast<long long>(R), static_cast<long long>(K));
  if (K % kGroup) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "K = %lld is not a multiple of 128",
                              static_cast<long long>(K));
  if (R == 0) return W4A8_OK;
  if (!w_bf16 || !packed || !scales_bf16) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(w_bf16) || !aligned16(packed) || !aligned16(scales_bf16))
    return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_pack_int4_channel(w_bf16, R, K, packed, scales_bf16, di.sms,
                                             static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "pack_int4_channel launch");
}

w4a8_status w4a8_prepare_experts_channel_b200(const int32_t* packed, int64_t E, int64_t rows,
                                              int64_t K, int32_t* packed_out,
                                              int32_t* nibble_sums, void* stream) {
  if (E < 0 || rows < 0 || K <= 0)
    return fail(W4A8_ERR_INVALID_ARG, "E = %lld, rows = %lld, K = %lld", static_cast<long long>(E),
                static_cast<long long>(rows), static_cast<long long>(K));
  if (K % kGroup) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "K = %lld is not a multiple of 128",
                              static_cast<long long>(K));
  const int64_t R = E * rows, nwords = R * (K / 8);
  if (nwords == 0) return W4A8_OK;
  if (!packed || !packed_out || !nibble_sums) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer");
  for (const void* p : {static_cast<const void*>(packed), static_cast<const void*>(packed_out),
                        static_cast<const void*>(nibble_sums)})
    if (!aligned16(p)) return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (packed != packed_out && packed < packed_out + nwords && packed_out < packed + nwords)
    return fail(W4A8_ERR_INVALID_ARG, "packed and packed_out overlap without being the same buffer");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the sums do not depend on the nibble order: take them before an in-place repack
  cudaError_t err = launch_nibble_row_sum(packed, R, K / 8, nibble_sums, di.sms, s);
  if (err == cudaSuccess) err = launch_repack_int4_b200(packed, nwords, packed_out, di.sms, s);
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "prepare_experts_channel launch");
}

w4a8_status w4a8_quant_fp8_block(const void* w_bf16, int64_t R, int64_t K, uint8_t* codes,
                                 float* scales, void* stream) {
  if (R < 0 || K < 0) return fail(W4A8_ERR_INVALID_ARG, "R = %lld, K = %lld",
                                  static_cast<long long>(R), static_cast<long long>(K));
  if (R % kGroup || K % kGroup)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "R = %lld and K = %lld must be multiples of 128",
                static_cast<long long>(R), static_cast<long long>(K));
  if (R == 0 || K == 0) return W4A8_OK;
  if (R / kGroup > 65535) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "R / 128 exceeds 65535");
  if (!w_bf16 || !codes || !scales) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(scales))
    return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_quant_fp8_block(w_bf16, R, K, codes, scales,
                                           static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "quant_fp8_block launch");
}

w4a8_status w4a8_quant_act_fp8_group(const void* x_bf16, int64_t T, int64_t H, uint8_t* codes,
                                     float* scales, void* stream) {
  if (T < 0 || H <= 0) return fail(W4A8_ERR_INVALID_ARG, "T = %lld, H = %lld",
                                   static_cast<long long>(T), static_cast<long long>(H));
  if (H % kGroup) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "H = %lld is not a multiple of 128",
                              static_cast<long long>(H));
  if (T == 0) return W4A8_OK;
  if (!x_bf16 || !codes || !scales) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales))
    return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_act_quant_group(x_bf16, nullptr, T, H, codes, scales, di.sms,
                                           static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "quant_act_fp8_group launch");
}

size_t w4a8_shared_expert_workspace_size(int64_t T, int64_t H, int64_t I) {
  if (T < 0 || H <= 0 || I <= 0) return 0;
  Carver c(nullptr);
  carve_shared(c, T, H, I, false);
  return c.off + 256;
}

w4a8_status w4a8_shared_expert_forward(const void* hidden_bf16, const uint8_t* w13_codes,
                                       const float* w13_scales, const uint8_t* w2_codes,
                                       const float* w2_scales, int64_t T, int64_t H, int64_t I,
                                       float* y, void* workspace, size_t workspace_bytes,
                                       const w4a8_shared_aux* aux, void* stream) {
  if (w4a8_status st = check_shared_shape(T, H, I)) return st;
  if (T == 0) return W4A8_OK;
  const void* ptrs[] = {hidden_bf16, w13_codes, w13_scales, w2_codes, w2_scales, y, workspace};
  for (const void* p : ptrs) {
    if (!p) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(p)) return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  const size_t need = w4a8_shared_expert_workspace_size(T, H, I);
  if (workspace_bytes < need)
    return fail(W4A8_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu", workspace_bytes, need);
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  Carver c(workspace);
  const SharedBufs b = carve_shared(c, T, H, I, false);
  return shared_forward_impl(hidden_bf16, w13_codes, w13_scales, w2_codes, w2_scales, T, H, I, y,
                             b, aux, di, static_cast<cudaStream_t>(stream));
}

size_t w4a8_moe_shared_workspace_size(int64_t T, int64_t H, int64_t I, int32_t E, int32_t k,
                                      int64_t I_shared) {
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1 || I_shared <= 0) return 0;
  Carver c(nullptr);
  carve_forward(c, T, H, I, E, k);
  carve_shared(c, T, H, I_shared, true);
  return c.off + 256;
}

w4a8_status w4a8_moe_forward_shared(const void* hidden_bf16, const float* logits,
                                    const int32_t* w13_packed, const void* w13_scales,
                                    const int32_t* w2_packed, const void* w2_scales,
                                    const uint8_t* ws13_codes, const float* ws13_scales,
                                    const uint8_t* ws2_codes, const float* ws2_scales,
                                    int64_t T, int64_t H, int64_t I, int64_t I_shared, int32_t E,
                                    int32_t k, void* out_bf16, void* workspace,
                                    size_t workspace_bytes, const w4a8_moe_aux* aux,
                                    const w4a8_shared_aux* shared_aux, void* stream) {
  const SharedExpert sh{ws13_codes, ws13_scales, ws2_codes, ws2_scales, I_shared, shared_aux};
  return moe_forward_impl(hidden_bf16, logits, w13_packed, w13_scales, w2_packed, w2_scales, T, H,
                          I, E, k, out_bf16, workspace, workspace_bytes, aux, stream, nullptr,
                          &sh);
}

// ---------------------------------------------------------------- expert parallelism

w4a8_status w4a8_moe_route_topk(const float* logits, int64_t T, int32_t E, int32_t k,
                                int32_t* topk_ids, float* topk_w, void* stream) {
  if (w4a8_status st = check_route_args(logits, T, E, k)) return st;
  if (T == 0) return W4A8_OK;
  if (!topk_ids || !topk_w) return fail(W4A8_ERR_INVALID_ARG, "NULL output pointer");
  if (!aligned16(topk_ids) || !aligned16(topk_w))
    return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_route_topk(logits, T, E, k, topk_ids, topk_w,
                                      static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "route_topk launch");
}

size_t w4a8_moe_experts_workspace_size(int64_t T, int64_t H, int64_t I, int32_t e_count,
                                       int32_t k) {
  if (T < 0 || H <= 0 || I <= 0 || e_count < 1 || k < 1) return 0;
  Carver c(nullptr);
  carve_forward(c, T, H, I, e_count, k);
  return c.off + 256;
}

w4a8_status w4a8_moe_forward_experts(const uint8_t* act_codes, const float* act_scales,
                                     const int32_t* topk_ids, const float* topk_w, int64_t T,
                                     int64_t H, int64_t I, int32_t E, int32_t k,
                                     int32_t e_begin, int32_t e_count,
                                     const int32_t* w13_packed, const void* w13_scales,
                                     const int32_t* w2_packed, const void* w2_scales,
                                     float* partial_out, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (T < 0) return fail(W4A8_ERR_INVALID_ARG, "T = %lld < 0", static_cast<long long>(T));
  if (E < 1 || E > kMaxExperts)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "E = %d outside [1, %d]", E, kMaxExperts);
  if (k < 1 || k > E || k > kMaxTopK)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "k = %d outside [1, min(E, %d)]", k, kMaxTopK);
  if (e_begin < 0 || e_count < 1 || e_begin + static_cast<int64_t>(e_count) > E)
    return fail(W4A8_ERR_INVALID_ARG, "expert range [%d, %d + %d) is not inside [0, %d)", e_begin,
                e_begin, e_count, E);
  if (T * static_cast<int64_t>(k) > INT32_MAX)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "T * k exceeds 2^31 - 1");
  if (H <= 0 || I <= 0 || H % kGroup || I % kGroup)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "H = %lld and I = %lld must be positive multiples of 128",
                static_cast<long long>(H), static_cast<long long>(I));
  if (H / kGroup > kMaxGroups || I / kGroup > kMaxGroups)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "H = %lld, I = %lld: at most %d groups of 128 per row",
                static_cast<long long>(H), static_cast<long long>(I), kMaxGroups);
  if (static_cast<int64_t>(e_count) * 2 * I > INT32_MAX || static_cast<int64_t>(e_count) * H > INT32_MAX)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "e_count * rows exceeds 2^31 - 1");
  if (T == 0) return W4A8_OK;
  const void* ptrs[] = {act_codes, act_scales, topk_ids, topk_w, w13_packed, w13_scales,
                        w2_packed, w2_scales, partial_out, workspace};
  for (const void* p : ptrs) {
    if (!p) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(p)) return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  const size_t need = w4a8_moe_experts_workspace_size(T, H, I, e_count, k);
  if (workspace_bytes < need)
    return fail(W4A8_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu", workspace_bytes, need);
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  int* latch = nullptr;
  if (cudaError_t err = device_error_latch(&latch)) return cuda_fail(err, "device error latch");
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  Carver c(workspace);
  ForwardBufs b = carve_forward(c, T, H, I, e_count, k);
  const int64_t A = T * k;   // rows of the buffers: every slot could be local
  // the shape by the expected local load, which is the whole layer's per-expert load
  const bool decode = A <= static_cast<int64_t>(kDecodeTokensPerExpert) * E;
  const bool split = split_tiles(A, E);
  const int tile_n = split ? kTileNDecode : grouped_gemm_tile_n(decode);
  const bool parts = !split && grouped_gemm_uses_sum_parts(decode);
  SplitTiles st;
  if (split) {
    st.wide_min = kTileNDecode;
    st.tile_n_wide = kTileNPrefill;
    st.tile_prefix_wide = b.route.tile_prefix_wide;
  }

  CUtensorMap tw1, ta1, tw2, ta2, ts1, ts2, tg1, tg2;
  if (w4a8_status st = encode_u8_2d(&tw1, w13_packed, static_cast<uint64_t>(H / 2),
                                    static_cast<uint64_t>(e_count) * 2 * I, 64, 64,
                                    CU_TENSOR_MAP_SWIZZLE_64B))
    return st;
  if (w4a8_status st = encode_u8_2d(&ta1, b.perm_codes, static_cast<uint64_t>(H),
                                    static_cast<uint64_t>(A), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&tw2, w2_packed, static_cast<uint64_t>(I / 2),
                                    static_cast<uint64_t>(e_count) * H, 64, 128,
                                    CU_TENSOR_MAP_SWIZZLE_64B))
    return st;
  if (w4a8_status st = encode_u8_2d(&ta2, b.inter_codes, static_cast<uint64_t>(I),
                                    static_cast<uint64_t>(A), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&tg1, b.act_parts, static_cast<uint64_t>(2 * sum_parts_ld(H)),
                                    static_cast<uint64_t>(A), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&tg2, b.inter_parts,
                                    static_cast<uint64_t>(2 * sum_parts_ld(I)),
                                    static_cast<uint64_t>(A), 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return st;
  if (w4a8_status st = encode_u8_2d(&ts1, w13_scales, static_cast<uint64_t>(2 * I) * 2,
                                    static_cast<uint64_t>(e_count) * (H / kGroup), 128,
                                    static_cast<uint32_t>(H / kGroup), CU_TENSOR_MAP_SWIZZLE_NONE))
    return st;
  if (w4a8_status st = encode_u8_2d(&ts2, w2_scales, static_cast<uint64_t>(H) * 2,
                                    static_cast<uint64_t>(e_count) * (I / kGroup), 256,
                                    static_cast<uint32_t>(I / kGroup), CU_TENSOR_MAP_SWIZZLE_NONE))
    return st;

  cudaError_t err = cudaSuccess;
#define W4A8_STEP(call, what)                              \
  do {                                                     \
    err = (call);                                          \
    if (err != cudaSuccess) return cuda_fail(err, what);   \
  } while (0)
  // the local experts' segments of all T tokens; rows_total = expert_offsets[e_count]
  W4A8_STEP(launch_route_local(topk_ids, T, E, k, e_begin, e_count, b.expert_offsets,
                               b.sorted_token_ids, b.row_of, b.route.block_counts,
                               b.route.block_base, b.route.tile_prefix, tile_n, b.row_amax, latch,
                               di.sms, s, st),
            "local routing launch");
  const int32_t* rows_total = b.expert_offsets + e_count;
  W4A8_STEP(launch_ep_gather(act_codes, T, H, b.sorted_token_ids, rows_total, A, b.perm_codes,
                             parts ? nullptr : b.act_gsum, parts ? b.act_parts : nullptr, di.sms, s),
            "dispatch gather launch");

  GemmArgs g1{};
  g1.K = static_cast<int>(H);
  g1.n_rows = static_cast<int>(2 * I);
  g1.half_rows = static_cast<int>(I);
  g1.E = e_count;
  g1.expert_offsets = b.expert_offsets;
  g1.tile_prefix = b.route.tile_prefix;
  g1.row_tokens = b.sorted_token_ids;
  g1.act_scale = act_scales;
  g1.act_gsum = b.act_gsum;
  g1.wscale = w13_scales;
  g1.out = b.h;
  g1.out_ld = I;
  g1.row_amax = b.row_amax;
  g1.act_rows = T;
  g1.timeout_ns = wait_timeout_ns();
  g1.nb_fastest = tile_order_nb_fastest(decode);
  g1.n_seg_rows = A;
  g1.n_tokens = T;
  if (split) {
    g1.nb_fastest = tile_order_nb_fastest(true);
    W4A8_STEP(launch_grouped_gemm_split(true, tw1, ta1, ts1, tg1, g1, b.route.tile_prefix_wide,
                                        di.sms, s),
              "gate/up GEMM launch");
  } else {
    W4A8_STEP(launch_grouped_gemm(true, decode, tw1, ta1, ts1, tg1, g1, di.sms, s),
              "gate/up GEMM launch");
  }
  W4A8_STEP(launch_inter_quant(b.h, b.row_amax, A, I, b.inter_codes, b.inter_scales,
                               parts ? nullptr : b.inter_gsum, di.sms, s, nullptr,
                               parts ? b.inter_parts : nullptr, rows_total),
            "intermediate quant launch");
  GemmArgs g2 = g1;
  g2.K = static_cast<int>(I);
  g2.n_rows = static_cast<int>(H);
  g2.half_rows = 0;
  g2.row_tokens = nullptr;
  g2.act_scale = b.inter_scales;
  g2.act_gsum = b.inter_gsum;
  g2.wscale = w2_scales;
  g2.out = b.y;
  g2.out_ld = H;
  g2.row_amax = nullptr;
  g2.act_rows = A;
  if (split) {
    W4A8_STEP(launch_grouped_gemm_split(false, tw2, ta2, ts2, tg2, g2, b.route.tile_prefix_wide,
                                        di.sms, s),
              "down GEMM launch");
  } else {
    W4A8_STEP(launch_grouped_gemm(false, decode, tw2, ta2, ts2, tg2, g2, di.sms, s),
              "down GEMM launch");
  }
  W4A8_STEP(launch_combine(b.y, b.row_of, topk_w, T, H, k, nullptr, di.sms, s, nullptr,
                           partial_out),
            "partial combine launch");
#undef W4A8_STEP
  return W4A8_OK;
}

w4a8_status w4a8_cast_f32_bf16(const float* x, int64_t n, void* out_bf16, void* stream) {
  if (n < 0) return fail(W4A8_ERR_INVALID_ARG, "n = %lld < 0", static_cast<long long>(n));
  if (n % 8) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "n = %lld is not a multiple of 8",
                         static_cast<long long>(n));
  if (n == 0) return W4A8_OK;
  if (!x || !out_bf16) return fail(W4A8_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(x) || !aligned16(out_bf16))
    return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_cast_bf16(x, n, out_bf16, di.sms, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "cast launch");
}

w4a8_status w4a8_ep_dispatch_plan(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E,
                                  int32_t n_ranks, int32_t* send_counts, int32_t* send_rows,
                                  int64_t send_rows_capacity, int32_t* pos, void* stream) {
  if (T < 0 || k < 1 || E < 1)
    return fail(W4A8_ERR_INVALID_ARG, "T = %lld, k = %d, E = %d", static_cast<long long>(T), k, E);
  if (n_ranks < 1 || n_ranks > kEpMaxRanks)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "n_ranks = %d outside [1, %d]", n_ranks, kEpMaxRanks);
  if (!send_counts || (T > 0 && (!topk_ids || !send_rows || !pos)))
    return fail(W4A8_ERR_INVALID_ARG, "NULL pointer argument");
  if (T > INT32_MAX / n_ranks)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "T * n_ranks exceeds int32 indices");
  if (send_rows_capacity < T * std::min<int64_t>(k, n_ranks))
    return fail(W4A8_ERR_INVALID_ARG, "send_rows_capacity %lld < T * min(k, n_ranks) = %lld",
                static_cast<long long>(send_rows_capacity),
                static_cast<long long>(T * std::min<int64_t>(k, n_ranks)));
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_ep_plan(topk_ids, T, k, E, n_ranks, send_counts, send_rows, pos,
                                   static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "dispatch plan launch");
}

w4a8_status w4a8_ep_gather_rows(const uint8_t* codes, const float* scales, const int32_t* topk_ids,
                                const float* topk_w, int64_t T, int64_t H, int32_t k,
                                const int32_t* send_rows, int64_t n_rows, uint8_t* codes_out,
                                float* scales_out, int32_t* ids_out, float* w_out, void* stream) {
  if (T < 0 || H <= 0 || k < 1 || n_rows < 0)
    return fail(W4A8_ERR_INVALID_ARG, "T = %lld, H = %lld, k = %d, n_rows = %lld",
                static_cast<long long>(T), static_cast<long long>(H), k,
                static_cast<long long>(n_rows));
  if (H % 16) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "H = %lld is not a multiple of 16",
                          static_cast<long long>(H));
  if (n_rows == 0) return W4A8_OK;
  if (!codes || !scales || !topk_ids || !topk_w || !send_rows || !codes_out || !scales_out ||
      !ids_out || !w_out)
    return fail(W4A8_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(codes) || !aligned16(codes_out))
    return fail(W4A8_ERR_INVALID_ARG, "codes pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_ep_gather_rows(codes, scales, topk_ids, topk_w, T, H, k, send_rows,
                                          n_rows, codes_out, scales_out, ids_out, w_out, di.sms,
                                          static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "row gather launch");
}

w4a8_status w4a8_ep_combine_rows(const float* back, int64_t n_rows, int64_t H, const int32_t* pos,
                                 int64_t T, int32_t n_ranks, void* out_bf16, void* stream) {
  if (T < 0 || H <= 0 || n_rows < 0)
    return fail(W4A8_ERR_INVALID_ARG, "T = %lld, H = %lld, n_rows = %lld",
                static_cast<long long>(T), static_cast<long long>(H),
                static_cast<long long>(n_rows));
  if (n_ranks < 1 || n_ranks > kEpMaxRanks)
    return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "n_ranks = %d outside [1, %d]", n_ranks, kEpMaxRanks);
  if (H % 8) return fail(W4A8_ERR_UNSUPPORTED_SHAPE, "H = %lld is not a multiple of 8",
                         static_cast<long long>(H));
  if (T == 0) return W4A8_OK;
  if (!pos || !out_bf16 || (n_rows > 0 && !back))
    return fail(W4A8_ERR_INVALID_ARG, "NULL pointer argument");
  if ((back && !aligned16(back)) || !aligned16(out_bf16))
    return fail(W4A8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceInfo di;
  if (w4a8_status st = device_info(&di)) return st;
  cudaError_t err = launch_ep_combine_rows(back, n_rows, H, pos, T, n_ranks, out_bf16, di.sms,
                                           static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? W4A8_OK : cuda_fail(err, "combine rows launch");
}

}  // extern "C"

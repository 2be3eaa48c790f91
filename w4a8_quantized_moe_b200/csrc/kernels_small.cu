// kernels_small.cu - the HBM-bound and latency-bound steps of the layer:
// per-token FP8 activation quantisation, INT4 RTN packing, top-k routing and
// the expert permutation, the intermediate requantisation, the combine.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>

#include "internal.h"

namespace w4a8 {

// Bounds checks of routing-derived indices (the debug build, compiled with
// W4A8_DEBUG_BOUNDS=1): an index outside its buffer raises the device latch's
// index bit and the access is skipped.  The release build compiles them out.
#if W4A8_DEBUG_BOUNDS
__device__ int* g_debug_latch = nullptr;
#define W4A8_IN_BOUNDS(cond) \
  ((cond) ? true : (atomicOr(::w4a8::g_debug_latch, ::w4a8::kDeviceErrorIndex), false))
#else
#define W4A8_IN_BOUNDS(cond) true
#endif

namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ float absmax8(uint4 c) {
  float m = fmaxf(fabsf(bf16_lo(c.x)), fabsf(bf16_hi(c.x)));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(c.y)), fabsf(bf16_hi(c.y))));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(c.z)), fabsf(bf16_hi(c.z))));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(c.w)), fabsf(bf16_hi(c.w))));
  return m;
}

// Two floats -> two E4M3 codes (first in the low byte), nearest-even, saturating.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Eight values / scale -> eight E4M3 codes (little-endian in a uint2).
__device__ __forceinline__ uint2 quant8(const float (&v)[8], float scale) {
  if (scale == 0.0f) return make_uint2(0u, 0u);
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    c[i] = e4m3x2(__fdiv_rn(v[2 * i], scale), __fdiv_rn(v[2 * i + 1], scale));
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// 8 values -> 8 offset-binary INT8 codes (byte = code + 128), code =
// clamp(rint(float32(v / scale)), -127, 127); scale 0 -> code 0.  The grouped
// GEMM multiplies unsigned bytes, so the codes are stored offset by 128.
__device__ __forceinline__ uint2 quant8_i8(const float (&v)[8], float scale) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int c = 0;
    if (scale != 0.0f) c = static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(v[i], scale)), -127.0f), 127.0f));
    b[i] = static_cast<uint32_t>(c + 128);
  }
  return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                    b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
}

// Sum of the 8 bytes of a uint2, as unsigned bytes (the unsigned dp4a).
__device__ __forceinline__ int sum8_u8(uint2 q) {
  return static_cast<int>(__dp4a(q.x, 0x01010101u, __dp4a(q.y, 0x01010101u, 0u)));
}

// Sum of the E4M3 values of the eight codes in c (low byte first).
__device__ __forceinline__ float sum8_e4m3(uint2 c) {
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t pair = static_cast<uint16_t>(((i < 2 ? c.x : c.y) >> (16 * (i & 1))) & 0xffffu);
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    s += f.x;
    s += f.y;
  }
  return s;
}

// A group sum as three bf16 parts, p0 + p1 + p2 = S to ~2^-27 |S| (each
// remainder is exact in FP32), at columns g, gp + g, 2 gp + g of `row`; the
// writer of the last group also zeroes the padding columns G .. gp - 1.
__device__ __forceinline__ void store_sum_parts(uint16_t* row, float S, int g, int G, int gp) {
  const __nv_bfloat16 p0 = __float2bfloat16_rn(S);
  const float r1 = S - __bfloat162float(p0);
  const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(p1);
  const __nv_bfloat16 p2 = __float2bfloat16_rn(r2);
  row[g] = __bfloat16_as_ushort(p0);
  row[gp + g] = __bfloat16_as_ushort(p1);
  row[2 * gp + g] = __bfloat16_as_ushort(p2);
  if (g == G - 1)
    for (int z = G; z < gp; ++z) row[z] = row[gp + z] = row[2 * gp + z] = 0;
}

__device__ __forceinline__ void unpack8(uint4 c, float (&v)[8]) {
  v[0] = bf16_lo(c.x); v[1] = bf16_hi(c.x); v[2] = bf16_lo(c.y); v[3] = bf16_hi(c.y);
  v[4] = bf16_lo(c.z); v[5] = bf16_hi(c.z); v[6] = bf16_lo(c.w); v[7] = bf16_hi(c.w);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// ---------------------------------------------------------------- activation quant
// One CTA per token row (grid-stride): absmax over the row, scale = absmax/448,
// codes = E4M3(x / scale).  Up to kAqCache 16-byte chunks per thread stay in
// registers between the two passes; longer rows are re-read (L1/L2 hits).
// Optionally also the sum of the E4M3 values (codes decoded, without the
// scale) of every 128-wide group, which the grouped GEMM needs because it
// feeds the weights to the MMA as q + 8 (see grouped_gemm.cu): 16 chunks of 8
// make a group, held by 16 consecutive threads.
constexpr int kAqThreads = 256;
constexpr int kAqCache = 4;

template <bool kInt8>
__global__ void __launch_bounds__(kAqThreads) act_quant_kernel(const __nv_bfloat16* __restrict__ x,
                                                               int64_t T, int64_t H,
                                                               uint8_t* __restrict__ codes,
                                                               float* __restrict__ scales,
                                                               float* __restrict__ gsum,
                                                               const int32_t* __restrict__ row_of,
                                                               int k,
                                                               uint8_t* __restrict__ perm,
                                                               int32_t* __restrict__ row_sum,
                                                               uint16_t* __restrict__ parts) {
  __shared__ float red[kAqThreads / 32];
  __shared__ int ired[kAqThreads / 32];
  __shared__ int64_t dst_rows[kMaxTopK];
  const int64_t nchunk = H / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(x + t * H);
    uint4 cache[kAqCache];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kAqCache; ++i) {
      const int64_t c = threadIdx.x + static_cast<int64_t>(i) * kAqThreads;
      if (c < nchunk) {
        cache[i] = __ldg(row + c);
        amax = fmaxf(amax, absmax8(cache[i]));
      }
    }
    for (int64_t c = threadIdx.x + static_cast<int64_t>(kAqCache) * kAqThreads; c < nchunk;
         c += kAqThreads)
      amax = fmaxf(amax, absmax8(__ldg(row + c)));
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    if (perm && threadIdx.x < k) {
      int64_t r = __ldg(row_of + t * k + threadIdx.x);
      if (!W4A8_IN_BOUNDS(r >= 0 && r < T * k)) r = -1;
      dst_rows[threadIdx.x] = r;
    }
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < kAqThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    const float scale = __fdiv_rn(amax, kInt8 ? 127.0f : 448.0f);
    if (threadIdx.x == 0) scales[t] = scale;
    uint2* out = reinterpret_cast<uint2*>(codes + t * H);
    float* gs = !kInt8 && gsum ? gsum + t * (H / kGroup) : nullptr;
    const bool want_sums = !kInt8 && (gsum || parts);
    const int G = static_cast<int>(H / kGroup);
    const int gp = (G + 15) / 16 * 16;
    int isum = 0;  // INT8: this thread's share of the row's offset-binary code sum
    // Every thread runs every chunk slot (the slot bounds are uniform) so that
    // the 16-lane group reductions see full warps.
    auto emit = [&](int64_t c, const uint4& raw) {
      float part = 0.0f;
      if (c < nchunk) {
        float v[8];
        unpack8(raw, v);
        const uint2 q = kInt8 ? quant8_i8(v, scale) : quant8(v, scale);
        out[c] = q;
        if (perm)  // the token's codes again at each of its k segment rows
          for (int j = 0; j < k; ++j)
            if (dst_rows[j] >= 0) reinterpret_cast<uint2*>(perm + dst_rows[j] * H)[c] = q;
        if (kInt8) isum += sum8_u8(q);
        if (want_sums) part = sum8_e4m3(q);
      }
      if (want_sums) {
        part += __shfl_xor_sync(kFull, part, 8);
        part += __shfl_xor_sync(kFull, part, 4);
        part += __shfl_xor_sync(kFull, part, 2);
        part += __shfl_xor_sync(kFull, part, 1);
        if (c < nchunk && (c & 15) == 0) {
          if (gs) gs[c >> 4] = part;
          if (parts)
            for (int j = 0; j < k; ++j)
              if (dst_rows[j] >= 0)
                store_sum_parts(parts + dst_rows[j] * sum_parts_ld(H), part, static_cast<int>(c >> 4), G, gp);
        }
      }
    };
#pragma unroll
    for (int i = 0; i < kAqCache; ++i) {
      if (static_cast<int64_t>(i) * kAqThreads >= nchunk) break;
      emit(threadIdx.x + static_cast<int64_t>(i) * kAqThreads, cache[i]);
    }
    for (int64_t base = static_cast<int64_t>(kAqCache) * kAqThreads; base < nchunk;
         base += kAqThreads) {
      const int64_t c = base + threadIdx.x;
      emit(c, c < nchunk ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u));
    }
    if (kInt8) {  // exact integer row sum of the offset-binary codes
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(kFull, isum, o);
      if (lane == 0) ired[warp] = isum;
      __syncthreads();
      if (threadIdx.x == 0) {
        int tot = 0;
        for (int w = 0; w < kAqThreads / 32; ++w) tot += ired[w];
        row_sum[t] = tot;
      }
    }
    __syncthreads();  // red[] and ired[] are reused by the next row
  }
}

// ---------------------------------------------------------------- INT4 pack
// One warp per group of 128 weights (grid-stride).  Lane l holds elements
// 4l..4l+3; q = clamp(rint(w / s), -8, 7); lanes 2i and 2i+1 form word i
// (nibbles little-endian along K).
//   kClip = false: s = bf16(absmax / 7) (round-to-nearest);
//   kClip = true:  the per-group MSE clip search over the 11 shrink ratios
//     r = 1.00, 0.97, ..., 0.70 (GLM-5.3-W4A8 model card, "quantisation
//     method"): candidate s_r = bf16(float32(absmax * r) / 7); the squared
//     error of each candidate is summed in float64 in a fixed order (each lane
//     sums its 4 values in sequence, then five xor-pairwise exchanges), with
//     explicitly rounded double operations, so the arg-min is a deterministic
//     function of the weights; the first (largest) ratio with the least error
//     is kept.
template <bool kClip>
__global__ void __launch_bounds__(256) pack_int4_kernel(const __nv_bfloat16* __restrict__ w,
                                                        int64_t R, int64_t K,
                                                        int32_t* __restrict__ packed,
                                                        __nv_bfloat16* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t groups_per_row = K / kGroup;
  const int64_t ngroups = R * groups_per_row;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t g = warp_global; g < ngroups; g += nwarps) {
    const int64_t r = g / groups_per_row, gi = g - r * groups_per_row;
    const __nv_bfloat16* src = w + r * K + gi * kGroup + lane * 4;
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src));
    float v[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    amax = warp_max(amax);
    auto codes = [&](float s, int (&q)[4]) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        q[i] = s != 0.0f ? static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(v[i], s)), -8.0f), 7.0f))
                         : 0;
    };
    __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
    int q[4];
    codes(__bfloat162float(sb), q);
    if constexpr (kClip) {
      double best = 0.0;
      for (int ri = 0; ri < 11; ++ri) {
        const float r = static_cast<float>((100.0 - 3.0 * ri) / 100.0);
        const __nv_bfloat16 cb = __float2bfloat16_rn(__fdiv_rn(__fmul_rn(amax, r), 7.0f));
        const float c = __bfloat162float(cb);
        int qc[4];
        codes(c, qc);
        double e = 0.0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const double d = __dsub_rn(static_cast<double>(v[i]),
                                     __dmul_rn(static_cast<double>(qc[i]), static_cast<double>(c)));
          e = i == 0 ? __dmul_rn(d, d) : __dadd_rn(e, __dmul_rn(d, d));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) e = __dadd_rn(e, __shfl_xor_sync(kFull, e, off));
        if (ri == 0 || e < best) {  // every lane holds the same e: the choice is warp-uniform
          best = e;
          sb = cb;
#pragma unroll
          for (int i = 0; i < 4; ++i) q[i] = qc[i];
        }
      }
    }
    uint32_t nib = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) nib |= static_cast<uint32_t>(q[i] + 8) << (4 * i);
    const uint32_t hi = __shfl_down_sync(kFull, nib, 1);
    if ((lane & 1) == 0)
      packed[r * (K / 8) + gi * (kGroup / 8) + (lane >> 1)] = static_cast<int32_t>(nib | (hi << 16));
    if (lane == 0) scales[r * groups_per_row + gi] = sb;
  }
}

// ---------------------------------------------------------------- per-channel INT4 pack
// One CTA per row: s = bf16(absmax of the whole row / 7) (per-channel RTN),
// q = clamp(rint(w / s), -8, 7), 8 nibbles per word little-endian along K.
__global__ void __launch_bounds__(256) pack_int4_channel_kernel(const __nv_bfloat16* __restrict__ w,
                                                                int64_t R, int64_t K,
                                                                int32_t* __restrict__ packed,
                                                                __nv_bfloat16* __restrict__ scales) {
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nchunk = K / 8;
  for (int64_t r = blockIdx.x; r < R; r += gridDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(w + r * K);
    float amax = 0.0f;
    for (int64_t c = threadIdx.x; c < nchunk; c += blockDim.x) amax = fmaxf(amax, absmax8(__ldg(row + c)));
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
    const float sc = __bfloat162float(sb);
    if (threadIdx.x == 0) scales[r] = sb;
    for (int64_t c = threadIdx.x; c < nchunk; c += blockDim.x) {
      float v[8];
      unpack8(__ldg(row + c), v);
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int q =
            sc != 0.0f ? static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(v[i], sc)), -8.0f), 7.0f)) : 0;
        word |= static_cast<uint32_t>(q + 8) << (4 * i);
      }
      packed[r * nchunk + c] = static_cast<int32_t>(word);
    }
    __syncthreads();  // red[] is reused by the next row
  }
}

// Warp per row: sum of all stored nibbles u = q + 8 of the row (any nibble order).
__global__ void __launch_bounds__(256) nibble_row_sum_kernel(const uint32_t* __restrict__ packed,
                                                             int64_t R, int64_t words_per_row,
                                                             int32_t* __restrict__ sums) {
  const int lane = threadIdx.x & 31;
  const int64_t wg = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = wg; r < R; r += nw) {
    int acc = 0;
    for (int64_t i = lane; i < words_per_row; i += 32) {
      const uint32_t x = __ldg(packed + r * words_per_row + i);
      acc = static_cast<int>(__dp4a(x & 0x0F0F0F0Fu, 0x01010101u, static_cast<unsigned>(acc)));
      acc = static_cast<int>(__dp4a((x >> 4) & 0x0F0F0F0Fu, 0x01010101u, static_cast<unsigned>(acc)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    if (lane == 0) sums[r] = acc;
  }
}

// ---------------------------------------------------------------- routing
// Top-k per token, one warp per token: lane l holds the logits of experts
// l, l+32, ...; k rounds of a warp arg-max under the order (larger logit, then
// lower id).  Weights: softmax of the selected logits in float32.  Each
// selection also counts into block_counts[token / kRouteTok][expert] (global
// atomics; the launcher zeroes the counts first).
template <int NV>  // logits per lane (E <= 32 * NV)
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int64_t T,
                                                         int E, int k, int32_t* __restrict__ topk_ids,
                                                         float* __restrict__ topk_w,
                                                         int32_t* __restrict__ block_counts) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;  // warp-uniform
  const float* lt = logits + t * E;
  int32_t* counts = block_counts ? block_counts + (t / kRouteTok) * E : nullptr;
  float v[NV];
  uint32_t taken = 0;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int e = lane + 32 * q;
    if (e < E) v[q] = __ldg(lt + e);
    else { v[q] = -INFINITY; taken |= 1u << q; }
  }
  float myv = 0.0f, v0 = 0.0f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int e = lane + 32 * q;
      if (!((taken >> q) & 1u) && (v[q] > bv || (v[q] == bv && e < bi))) { bv = v[q]; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, o);
      const int oi = __shfl_xor_sync(kFull, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) {
      myv = bv;
      topk_ids[t * k + j] = bi;
      if (block_counts) atomicAdd(counts + bi, 1);
    }
    if (j == 0) v0 = bv;
  }
  const float ex = (lane < k) ? expf(myv - v0) : 0.0f;
  const float sum = warp_sum(ex);
  if (lane < k) topk_w[t * k + lane] = __fdiv_rn(ex, sum);
}

// Exclusive scan over the experts (one CTA of 1024 threads, thread = expert):
// per-block bases within each expert, expert offsets, GEMM tile prefix.
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh /*[32]*/, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = (lane < static_cast<int>(blockDim.x >> 5)) ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, s, o);
      if (lane >= o) s += y;
    }
    sh[lane] = s;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = x - v + (warp > 0 ? sh[warp - 1] : 0);
  *total = sh[(blockDim.x >> 5) - 1];
  __syncthreads();
  return excl;
}

// Split tiling (tile_prefix_wide != nullptr): experts with more than wide_min
// assignments get their tiles in tile_prefix_wide (tile_n_wide rows each) and
// none in tile_prefix, the others the reverse, so that two GEMM launches of
// different tile shapes cover disjoint experts.
__global__ void __launch_bounds__(1024) route_scan_kernel(const int32_t* __restrict__ block_counts,
                                                          int64_t nblk, int E, int tile_n,
                                                          int32_t* __restrict__ block_base,
                                                          int32_t* __restrict__ expert_offsets,
                                                          int32_t* __restrict__ tile_prefix,
                                                          int wide_min, int tile_n_wide,
                                                          int32_t* __restrict__ tile_prefix_wide) {
  __shared__ int sh[32];
  const int e = threadIdx.x;
  int running = 0;
  if (e < E) {
    int64_t b = 0;
    for (; b + 8 <= nblk; b += 8) {
      int c[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) c[u] = __ldg(block_counts + (b + u) * E + e);
#pragma unroll
      for (int u = 0; u < 8; ++u) { block_base[(b + u) * E + e] = running; running += c[u]; }
    }
    for (; b < nblk; ++b) {
      const int c = __ldg(block_counts + b * E + e);
      block_base[b * E + e] = running;
      running += c;
    }
  }
  int total = 0, total_tiles = 0;
  const int off = block_exclusive_scan(e < E ? running : 0, sh, &total);
  const bool wide = tile_prefix_wide != nullptr && running > wide_min;
  const int tiles = (e < E && !wide) ? (running + tile_n - 1) / tile_n : 0;
  const int toff = block_exclusive_scan(tiles, sh, &total_tiles);
  if (e < E) {
    expert_offsets[e] = off;
    tile_prefix[e] = toff;
    for (int64_t b = 0; b < nblk; ++b) block_base[b * E + e] += off;
  }
  if (e == 0) {
    expert_offsets[E] = total;
    tile_prefix[E] = total_tiles;
  }
  if (tile_prefix_wide != nullptr) {  // uniform: every thread takes part in the scan
    int total_wide = 0;
    const int wtiles = (e < E && wide) ? (running + tile_n_wide - 1) / tile_n_wide : 0;
    const int woff = block_exclusive_scan(wtiles, sh, &total_wide);
    if (e < E) tile_prefix_wide[e] = woff;
    if (e == 0) tile_prefix_wide[E] = total_wide;
  }
}

// Stable scatter: one CTA per routing block of 256 tokens, warp w owns tokens
// 32w..32w+31 of the block (lane = token).  mask[w][e] has bit l set when
// token l of chunk w chose expert e; the rank of a token among the block's
// tokens of expert e is the popcount of the earlier chunks' masks plus the
// bits below it in its own chunk's mask.
constexpr int kScatterWarps = kRouteTok / 32;

// Only experts e_lo .. e_lo + E - 1 get segments (E = the segment count; the
// whole layer passes e_lo = 0): an assignment to any other expert gets
// row_of = -1 and no row (expert parallelism: the experts of other ranks).
__global__ void __launch_bounds__(kRouteTok) route_scatter_kernel(
    const int32_t* __restrict__ topk_ids, int64_t T, int E, int k, int e_lo,
    const int32_t* __restrict__ block_base, int32_t* __restrict__ sorted_token_ids,
    int32_t* __restrict__ row_of, uint32_t* __restrict__ row_amax) {
  extern __shared__ uint32_t mask[];  // [kScatterWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteTok + threadIdx.x;
  const bool valid = t < T;
  int ids[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    ids[j] = (valid && j < k) ? __ldg(topk_ids + t * k + j) - e_lo : -1;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (static_cast<unsigned>(ids[j]) < static_cast<unsigned>(E))
      atomicOr(&mask[warp * E + ids[j]], 1u << lane);
  __syncthreads();
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int32_t* base = block_base + static_cast<int64_t>(blockIdx.x) * E;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (valid && j < k) {
      const int e = ids[j];
      if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) {
        row_of[t * k + j] = -1;
        continue;
      }
      int rank = __popc(mask[warp * E + e] & lt_mask);
      for (int w = 0; w < warp; ++w) rank += __popc(mask[w * E + e]);
      const int row = base[e] + rank;
      if (!W4A8_IN_BOUNDS(row >= 0 && row < T * k)) {
        row_of[t * k + j] = -1;
        continue;
      }
      row_of[t * k + j] = row;
      sorted_token_ids[row] = static_cast<int32_t>(t);
      if (row_amax) row_amax[row] = 0u;
    }
  }
}

// Histogram of given expert ids for the experts e_lo .. e_lo + E_loc - 1 into
// block_counts[token / kRouteTok][e - e_lo] (thread per assignment; the
// launcher zeroes the counts).  An id outside [0, E_all) other than -1 (no
// expert) is a caller error: it raises the device latch's index bit and is
// left out.
__global__ void __launch_bounds__(256) route_ids_hist_kernel(const int32_t* __restrict__ topk_ids,
                                                             int64_t T, int k, int E_all, int e_lo,
                                                             int E_loc,
                                                             int32_t* __restrict__ block_counts,
                                                             int* __restrict__ latch) {
  const int64_t n = T * k;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = __ldg(topk_ids + i);
    if (e < -1 || e >= E_all) {
      atomicOr(latch, kDeviceErrorIndex);
      continue;
    }
    const int le = e - e_lo;
    if (e >= 0 && static_cast<unsigned>(le) < static_cast<unsigned>(E_loc))
      atomicAdd(block_counts + (i / k / kRouteTok) * E_loc + le, 1);
  }
}

// Expert-parallel dispatch: segment row r (r < expert_offsets[E_loc], read on
// the device) receives the E4M3 codes of token sorted_token_ids[r]; the sums
// of the E4M3 values of its 128-wide groups go to gsum [T, H / 128] (by token;
// several rows of one token write the same values) or, for the shapes that
// remove the nibble offset once per tile, to the row's three bf16 parts.
// One warp per row, 16 bytes per lane per step.
__global__ void __launch_bounds__(256) ep_gather_kernel(const uint8_t* __restrict__ codes,
                                                        int64_t T, int64_t H,
                                                        const int32_t* __restrict__ sorted_token_ids,
                                                        const int32_t* __restrict__ rows_total,
                                                        uint8_t* __restrict__ perm,
                                                        float* __restrict__ gsum,
                                                        uint16_t* __restrict__ parts) {
  const int lane = threadIdx.x & 31;
  const int64_t A = __ldg(rows_total);
  const int64_t nchunk = H / 16;                 // 16-byte chunks; 8 per 128-wide group
  const int G = static_cast<int>(H / kGroup);
  const int gp = (G + 15) / 16 * 16;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < A;
       r += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int64_t t = __ldg(sorted_token_ids + r);
    if (!W4A8_IN_BOUNDS(t >= 0 && t < T)) continue;   // warp-uniform
    const uint4* src = reinterpret_cast<const uint4*>(codes + t * H);
    uint4* dst = reinterpret_cast<uint4*>(perm + r * H);
    for (int64_t base = 0; base < nchunk; base += 32) {   // warp-uniform trip count
      const int64_t c = base + lane;
      float part = 0.0f;
      if (c < nchunk) {
        const uint4 v = __ldg(src + c);
        dst[c] = v;
        part = sum8_e4m3(make_uint2(v.x, v.y)) + sum8_e4m3(make_uint2(v.z, v.w));
      }
      part += __shfl_xor_sync(kFull, part, 4);
      part += __shfl_xor_sync(kFull, part, 2);
      part += __shfl_xor_sync(kFull, part, 1);
      if (c < nchunk && (c & 7) == 0) {
        if (gsum) gsum[t * G + (c >> 3)] = part;
        if (parts) store_sum_parts(parts + r * sum_parts_ld(H), part, static_cast<int>(c >> 3), G, gp);
      }
    }
  }
}

// float32 -> bf16, round to nearest even, 8 values per thread.
__global__ void __launch_bounds__(256) cast_bf16_kernel(const float* __restrict__ x, int64_t n8,
                                                        __nv_bfloat16* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(x) + 2 * i);
    const float4 b = __ldg(reinterpret_cast<const float4*>(x) + 2 * i + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t p[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
      p[q] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    reinterpret_cast<uint4*>(out)[i] = make_uint4(p[0], p[1], p[2], p[3]);
  }
}

// ---------------------------------------------------------------- intermediate requant
// 16 consecutive values of one segment row per thread: scale = amax_r / 448,
// codes = E4M3(h / scale), and the sum of the E4M3 values of each 128-wide
// group (8 consecutive threads).  Whole warps run every iteration so that
// the group reduction can use shuffles.
template <bool kInt8>
__global__ void __launch_bounds__(256) inter_quant_kernel(const float* __restrict__ h,
                                                          const uint32_t* __restrict__ row_amax,
                                                          int64_t A, int64_t I,
                                                          uint8_t* __restrict__ codes,
                                                          float* __restrict__ scales,
                                                          float* __restrict__ gsum,
                                                          int32_t* __restrict__ row_sum,
                                                          uint16_t* __restrict__ parts,
                                                          const int32_t* __restrict__ rows_dev) {
  const int64_t per_row = I / 16;
  const bool want_sums = !kInt8 && (gsum || parts);
  const int G = static_cast<int>(I / kGroup);
  const int gp = (G + 15) / 16 * 16;
  if (rows_dev) {  // the row count is known only on the device (expert parallelism)
    const int64_t a_dev = __ldg(rows_dev);
    A = a_dev < A ? a_dev : A;
  }
  const int64_t n = A * per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t n_iter = (n + stride - 1) / stride;
  for (int64_t k = 0; k < n_iter; ++k) {
    const int64_t i = k * stride + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const bool active = i < n;
    float part = 0.0f;
    int64_t r = 0, c = 0;
    if (active) {
      r = i / per_row;
      c = i - r * per_row;
      const float amax = __uint_as_float(__ldg(row_amax + r));
      const float scale = __fdiv_rn(amax, kInt8 ? 127.0f : 448.0f);
      if (c == 0) scales[r] = scale;
      const float4* src = reinterpret_cast<const float4*>(h + r * I + c * 16);
      uint2 out[2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const float4 a = __ldg(src + 2 * half), b = __ldg(src + 2 * half + 1);
        const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        out[half] = kInt8 ? quant8_i8(v, scale) : quant8(v, scale);
      }
      *reinterpret_cast<uint4*>(codes + r * I + c * 16) =
          make_uint4(out[0].x, out[0].y, out[1].x, out[1].y);
      if (kInt8) atomicAdd(row_sum + r, sum8_u8(out[0]) + sum8_u8(out[1]));  // exact, any order
      else if (want_sums) part = sum8_e4m3(out[0]) + sum8_e4m3(out[1]);
    }
    if (want_sums) {
      part += __shfl_xor_sync(kFull, part, 4);
      part += __shfl_xor_sync(kFull, part, 2);
      part += __shfl_xor_sync(kFull, part, 1);
      if (active && (c & 7) == 0) {
        if (gsum) gsum[r * (I / kGroup) + (c >> 3)] = part;
        if (parts) store_sum_parts(parts + r * sum_parts_ld(I), part, static_cast<int>(c >> 3), G, gp);
      }
    }
  }
}

// ---------------------------------------------------------------- FP8 block quantisers
// Weights: one CTA per 128 x 128 block (blockIdx.y: row block, blockIdx.x:
// column block); thread i reads rows i / 16 + 16 j (j < 8), 8 columns at
// (i % 16) * 8.  scale = float32(absmax / 448), codes = E4M3(w / scale).
__global__ void __launch_bounds__(256) quant_fp8_block_kernel(const __nv_bfloat16* __restrict__ w,
                                                              int64_t K, uint8_t* __restrict__ codes,
                                                              float* __restrict__ scales) {
  __shared__ float red[8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kGroup + tid / 16;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kGroup + (tid % 16) * 8;
  uint4 v[8];
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[j] = __ldg(reinterpret_cast<const uint4*>(w + (r0 + 16 * j) * K + c0));
    amax = fmaxf(amax, absmax8(v[j]));
  }
  amax = warp_max(amax);
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float scale = __fdiv_rn(amax, 448.0f);
  if (tid == 0) scales[static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x] = scale;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float f[8];
    unpack8(v[j], f);
    *reinterpret_cast<uint2*>(codes + (r0 + 16 * j) * K + c0) = quant8(f, scale);
  }
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  unpack8(__ldg(reinterpret_cast<const uint4*>(p)), f);
}
__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Activations (bf16 x or float32 h): one float32 scale per row and 128-wide
// group, scale = float32(absmax / 448).  8 values per thread; the 16
// consecutive threads of a group reduce the absmax with shuffles (whole warps
// run every iteration; H % 128 == 0 keeps a group inside one half-warp).
template <class TIn>
__global__ void __launch_bounds__(256) act_quant_group_kernel(const TIn* __restrict__ x, int64_t T,
                                                              int64_t H, uint8_t* __restrict__ codes,
                                                              float* __restrict__ scales) {
  const int64_t per_row = H / 8;
  const int64_t n = T * per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t n_iter = (n + stride - 1) / stride;
  for (int64_t it = 0; it < n_iter; ++it) {
    const int64_t i = it * stride + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const bool active = i < n;
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (active) load8(x + i * 8, f);
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 8));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 4));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    if (active) {
      const float scale = __fdiv_rn(amax, 448.0f);
      *reinterpret_cast<uint2*>(codes + i * 8) = quant8(f, scale);
      if ((i & 15) == 0) scales[i / 16] = scale;   // row-major [T, H / 128]
    }
  }
}

// Expert tables of a dense (one-expert) GEMM over T rows.
__global__ void dense_tables_kernel(int32_t* offsets, int32_t* tile_prefix, int32_t T, int tile_n) {
  if (threadIdx.x == 0) {
    offsets[0] = 0;
    offsets[1] = T;
    tile_prefix[0] = 0;
    tile_prefix[1] = (T + tile_n - 1) / tile_n;
  }
}

// ---------------------------------------------------------------- B200 weight layout
// Word-local nibble interleave: element j of each group of 8 moves from
// nibble j to nibble 2j (j < 4) or 2(j - 4) + 1 (j >= 4), so that w & 0x0F0F0F0F
// holds elements 0..3 one per byte and (w >> 4) & 0x0F0F0F0F elements 4..7.
// `in` may equal `out` (each thread reads its word before writing it).
__global__ void __launch_bounds__(256) repack_int4_b200_kernel(const uint32_t* in, int64_t nwords,
                                                               uint32_t* out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t w = in[i];
    uint32_t r = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t nib = (w >> (4 * j)) & 0xFu;
      const int p = j < 4 ? 2 * j : 2 * (j - 4) + 1;
      r |= nib << (4 * p);
    }
    out[i] = r;
  }
}

// [E, rows, G] -> [E, G, rows] (group-major weight scales).
__global__ void __launch_bounds__(256) transpose_scales_kernel(const uint16_t* __restrict__ in,
                                                               int64_t E, int64_t rows, int64_t G,
                                                               uint16_t* __restrict__ out) {
  const int64_t n = E * G * rows;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = i / (G * rows);
    const int64_t rem = i - e * G * rows;
    const int64_t g = rem / rows, r = rem - g * rows;
    out[i] = __ldg(in + (e * rows + r) * G + g);
  }
}

// ---------------------------------------------------------------- combine
// out[t, c..c+7] = bf16(sum_j w[t, j] * Y[row_of[t, j], c..c+7]) in slot order.
// kPartial: the float32 sum over the slots with a row (row_of >= 0: this
// rank's experts) instead, for the expert-parallel combine.
template <bool kPartial>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y,
                                                      const int32_t* __restrict__ row_of,
                                                      const float* __restrict__ topk_w, int64_t T,
                                                      int64_t H, int k,
                                                      const float* __restrict__ y_shared,
                                                      __nv_bfloat16* __restrict__ out,
                                                      float* __restrict__ out_f32) {
  const int64_t per_row = H / 8;
  const int64_t n = T * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_row, c = i - t * per_row;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int64_t r = __ldg(row_of + t * k + j);
      if (kPartial && r < 0) continue;
      if (!W4A8_IN_BOUNDS(r >= 0 && r < T * k)) continue;
      const float wj = __ldg(topk_w + t * k + j);
      const float4* src = reinterpret_cast<const float4*>(y + r * H + c * 8);
      const float4 a = __ldg(src), b = __ldg(src + 1);
      acc[0] = fmaf(wj, a.x, acc[0]); acc[1] = fmaf(wj, a.y, acc[1]);
      acc[2] = fmaf(wj, a.z, acc[2]); acc[3] = fmaf(wj, a.w, acc[3]);
      acc[4] = fmaf(wj, b.x, acc[4]); acc[5] = fmaf(wj, b.y, acc[5]);
      acc[6] = fmaf(wj, b.z, acc[6]); acc[7] = fmaf(wj, b.w, acc[7]);
    }
    if (y_shared) {  // the shared expert, added after the routed slots
      const float4* src = reinterpret_cast<const float4*>(y_shared + t * H + c * 8);
      const float4 a = __ldg(src), b = __ldg(src + 1);
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    if constexpr (kPartial) {
      float4* dst = reinterpret_cast<float4*>(out_f32 + t * H + c * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint32_t p[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        p[q] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      *reinterpret_cast<uint4*>(out + t * H + c * 8) = make_uint4(p[0], p[1], p[2], p[3]);
    }
  }
}

// ------------------------------------------- expert-parallel all-to-all(v)
// Dispatch by all-to-all(v): each rank sends each of its tokens once to every
// rank that owns one of the token's k experts, and adds the partial sums that
// come back.  Rank r of n owns a contiguous expert range; the first E % n
// ranks hold one more expert.
__device__ __forceinline__ int ep_owner(int e, int E, int n) {
  const int base = E / n, extra = E % n;
  const int cut = extra * (base + 1);              // experts of the larger ranks
  return e < cut ? e / (base + 1) : extra + (e - cut) / base;
}

// One CTA.  Pass 1 counts the tokens per rank; pass 2 walks the tokens in
// chunks of the block size and places each (token, rank) pair: rank-major,
// tokens ascending inside a rank (ballot prefix within a warp, a per-rank
// prefix over the warps, a running offset per rank across chunks).
constexpr int kPlanThreads = 1024;
__global__ void __launch_bounds__(kPlanThreads) ep_plan_kernel(const int32_t* __restrict__ ids,
                                                               int64_t T, int k, int E, int n,
                                                               int32_t* __restrict__ counts,
                                                               int32_t* __restrict__ rows,
                                                               int32_t* __restrict__ pos) {
  __shared__ int s_off[kEpMaxRanks];               // totals, then running offsets
  __shared__ int s_warp[kPlanThreads / 32][kEpMaxRanks];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < kEpMaxRanks) s_off[tid] = 0;
  __syncthreads();
  auto ranks_of = [&](int64_t t) -> uint64_t {     // the ranks token t goes to
    uint64_t m = 0;
    if (t < T)
      for (int j = 0; j < k; ++j) {
        const int e = __ldg(ids + t * k + j);
        if (e >= 0 && e < E) m |= 1ull << ep_owner(e, E, n);
      }
    return m;
  };
  for (int64_t c0 = 0; c0 < T; c0 += kPlanThreads) {
    const uint64_t m = ranks_of(c0 + tid);
    for (int r = 0; r < n; ++r) {
      const unsigned b = __ballot_sync(kFull, (m >> r) & 1u);
      if (lane == 0 && b) atomicAdd(&s_off[r], __popc(b));
    }
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int r = 0; r < n; ++r) {
      const int c = s_off[r];
      counts[r] = c;
      s_off[r] = acc;
      acc += c;
    }
  }
  __syncthreads();
  for (int64_t c0 = 0; c0 < T; c0 += kPlanThreads) {
    const int64_t t = c0 + tid;
    const uint64_t m = ranks_of(t);
    for (int r = 0; r < n; ++r) {
      const unsigned b = __ballot_sync(kFull, (m >> r) & 1u);
      if (lane == 0) s_warp[warp][r] = __popc(b);
    }
    __syncthreads();
    if (tid < n) {                                 // thread r: warp bases of rank r
      int acc = s_off[tid];
      for (int w = 0; w < kPlanThreads / 32; ++w) {
        const int c = s_warp[w][tid];
        s_warp[w][tid] = acc;
        acc += c;
      }
      s_off[tid] = acc;
    }
    __syncthreads();
    for (int r = 0; r < n; ++r) {
      const bool f = (m >> r) & 1u;
      const unsigned b = __ballot_sync(kFull, f);
      if (f) {
        const int p = s_warp[warp][r] + __popc(b & ((1u << lane) - 1u));
        rows[p] = static_cast<int32_t>(t);
        pos[t * n + r] = p;
      } else if (t < T) {
        pos[t * n + r] = -1;
      }
    }
    __syncthreads();                               // s_warp is refilled by the next chunk
  }
}

// Row i of the send buffers = row rows[i] of the rank's codes, scales, ids and
// weights.  One warp per row, 16 bytes of codes per lane per step.
__global__ void __launch_bounds__(256) ep_gather_rows_kernel(
    const uint8_t* __restrict__ codes, const float* __restrict__ scales,
    const int32_t* __restrict__ ids, const float* __restrict__ w, int64_t T, int64_t H, int k,
    const int32_t* __restrict__ rows, int64_t n_rows, uint8_t* __restrict__ codes_out,
    float* __restrict__ scales_out, int32_t* __restrict__ ids_out, float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int64_t nchunk = H / 16;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; i < n_rows;
       i += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int64_t t = __ldg(rows + i);
    if (!W4A8_IN_BOUNDS(t >= 0 && t < T)) continue;   // warp-uniform
    const uint4* src = reinterpret_cast<const uint4*>(codes + t * H);
    uint4* dst = reinterpret_cast<uint4*>(codes_out + i * H);
    for (int64_t c = lane; c < nchunk; c += 32) dst[c] = __ldg(src + c);
    for (int j = lane; j < k; j += 32) {
      ids_out[i * k + j] = __ldg(ids + t * k + j);
      w_out[i * k + j] = __ldg(w + t * k + j);
    }
    if (lane == 0) scales_out[i] = __ldg(scales + t);
  }
}

// out[t] = bf16(sum over ranks r ascending with pos[t, r] >= 0 of back[pos[t, r]]),
// float32 sums; a token that went nowhere gets zeros.  One thread per 8 columns.
__global__ void __launch_bounds__(256) ep_combine_rows_kernel(const float* __restrict__ back,
                                                              int64_t n_rows, int64_t H,
                                                              const int32_t* __restrict__ pos,
                                                              int64_t T, int n,
                                                              __nv_bfloat16* __restrict__ out) {
  const int64_t nc = H / 8;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < T * nc;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = idx / nc, c = idx - t * nc;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int r = 0; r < n; ++r) {
      const int64_t p = __ldg(pos + t * n + r);
      if (p < 0 || !W4A8_IN_BOUNDS(p < n_rows)) continue;
      const float4* src = reinterpret_cast<const float4*>(back + p * H + c * 8);
      const float4 a = __ldg(src), b = __ldg(src + 1);
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      q[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    *reinterpret_cast<uint4*>(out + t * H + c * 8) = make_uint4(q[0], q[1], q[2], q[3]);
  }
}

// Debug build: point g_debug_latch at the library's device error latch (once
// per device, before the first checked kernel).  Release build: nothing.
cudaError_t ensure_debug_latch() {
#if W4A8_DEBUG_BOUNDS
  static int* done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  int* latch = nullptr;
  err = device_error_latch(&latch);
  if (err != cudaSuccess) return err;
  if (dev < 64 && done[dev] == latch) return cudaSuccess;
  err = cudaMemcpyToSymbol(g_debug_latch, &latch, sizeof(latch));
  if (err == cudaSuccess && dev < 64) done[dev] = latch;
  return err;
#else
  return cudaSuccess;
#endif
}

inline int grid_for(int64_t work_items, int threads, int num_sms, int per_sm = 8) {
  int64_t g = (work_items + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms) * per_sm;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_act_quant(const void* x, int64_t T, int64_t H, uint8_t* codes, float* scales,
                             float* gsum, const int32_t* row_of, int k, uint8_t* perm, int num_sms,
                             cudaStream_t s, int32_t* int8_row_sum, uint16_t* sum_parts) {
  if (T == 0) return cudaSuccess;
  if (perm && (!row_of || k < 1 || k > kMaxTopK)) return cudaErrorInvalidValue;
  if (sum_parts && (!perm || int8_row_sum)) return cudaErrorInvalidValue;
  if (cudaError_t err = ensure_debug_latch()) return err;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int grid = static_cast<int>(T < cap ? T : cap);
  if (int8_row_sum)
    act_quant_kernel<true><<<grid, kAqThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), T, H,
                                                       codes, scales, nullptr, row_of, k, perm,
                                                       int8_row_sum, nullptr);
  else
    act_quant_kernel<false><<<grid, kAqThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), T, H,
                                                        codes, scales, gsum, row_of, k, perm,
                                                        nullptr, sum_parts);
  return cudaGetLastError();
}

cudaError_t launch_pack_int4(const void* w, int64_t R, int64_t K, int32_t* packed, void* scales,
                             bool clip_search, int num_sms, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  const int64_t ngroups = R * (K / kGroup);
  const int grid = grid_for(ngroups * 32, 256, num_sms, 16);
  if (clip_search)
    pack_int4_kernel<true><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), R, K,
                                                packed, static_cast<__nv_bfloat16*>(scales));
  else
    pack_int4_kernel<false><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), R, K,
                                                 packed, static_cast<__nv_bfloat16*>(scales));
  return cudaGetLastError();
}

cudaError_t launch_route(const float* logits, int64_t T, int E, int k, int32_t* topk_ids,
                         float* topk_w, int32_t* expert_offsets, int32_t* sorted_token_ids,
                         int32_t* row_of, int32_t* block_counts, int32_t* block_base,
                         int32_t* tile_prefix, int tile_n, uint32_t* row_amax_to_zero,
                         cudaStream_t s, const SplitTiles& split) {
  if (cudaError_t err = ensure_debug_latch()) return err;
  const int64_t nblk = route_blocks(T);
  if (nblk > 0) {
    cudaError_t err = cudaMemsetAsync(block_counts, 0,
                                      static_cast<size_t>(nblk) * E * sizeof(int32_t), s);
    if (err != cudaSuccess) return err;
    const int64_t grid = (T + 7) / 8;  // one warp per token, 8 per CTA
    const int nv = (E + 31) / 32;
    if (nv <= 1)
      route_topk_kernel<1><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
    else if (nv <= 2)
      route_topk_kernel<2><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
    else if (nv <= 4)
      route_topk_kernel<4><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
    else if (nv <= 8)
      route_topk_kernel<8><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
    else if (nv <= 16)
      route_topk_kernel<16><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
    else
      route_topk_kernel<32><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  route_scan_kernel<<<1, 1024, 0, s>>>(block_counts, nblk, E, tile_n, block_base,
                                       expert_offsets, tile_prefix, split.wide_min,
                                       split.tile_n_wide, split.tile_prefix_wide);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || nblk == 0) return err;
  const size_t smem = static_cast<size_t>(kScatterWarps) * E * sizeof(uint32_t);
  route_scatter_kernel<<<nblk, kRouteTok, smem, s>>>(topk_ids, T, E, k, 0, block_base,
                                                     sorted_token_ids, row_of, row_amax_to_zero);
  return cudaGetLastError();
}

cudaError_t launch_route_topk(const float* logits, int64_t T, int E, int k, int32_t* topk_ids,
                              float* topk_w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int64_t grid = (T + 7) / 8;
  const int nv = (E + 31) / 32;
  if (nv <= 1)
    route_topk_kernel<1><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, nullptr);
  else if (nv <= 2)
    route_topk_kernel<2><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, nullptr);
  else if (nv <= 4)
    route_topk_kernel<4><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, nullptr);
  else if (nv <= 8)
    route_topk_kernel<8><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, nullptr);
  else if (nv <= 16)
    route_topk_kernel<16><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, nullptr);
  else
    route_topk_kernel<32><<<grid, 256, 0, s>>>(logits, T, E, k, topk_ids, topk_w, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_route_local(const int32_t* topk_ids, int64_t T, int E_all, int k, int e_lo,
                               int E_loc, int32_t* expert_offsets, int32_t* sorted_token_ids,
                               int32_t* row_of, int32_t* block_counts, int32_t* block_base,
                               int32_t* tile_prefix, int tile_n, uint32_t* row_amax_to_zero,
                               int* latch, int num_sms, cudaStream_t s, const SplitTiles& split) {
  if (cudaError_t err = ensure_debug_latch()) return err;
  const int64_t nblk = route_blocks(T);
  if (nblk > 0) {
    cudaError_t err = cudaMemsetAsync(block_counts, 0,
                                      static_cast<size_t>(nblk) * E_loc * sizeof(int32_t), s);
    if (err != cudaSuccess) return err;
    route_ids_hist_kernel<<<grid_for(T * k, 256, num_sms), 256, 0, s>>>(
        topk_ids, T, k, E_all, e_lo, E_loc, block_counts, latch);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  route_scan_kernel<<<1, 1024, 0, s>>>(block_counts, nblk, E_loc, tile_n, block_base,
                                       expert_offsets, tile_prefix, split.wide_min,
                                       split.tile_n_wide, split.tile_prefix_wide);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || nblk == 0) return err;
  const size_t smem = static_cast<size_t>(kScatterWarps) * E_loc * sizeof(uint32_t);
  route_scatter_kernel<<<nblk, kRouteTok, smem, s>>>(topk_ids, T, E_loc, k, e_lo, block_base,
                                                     sorted_token_ids, row_of, row_amax_to_zero);
  return cudaGetLastError();
}

cudaError_t launch_ep_gather(const uint8_t* codes, int64_t T, int64_t H,
                             const int32_t* sorted_token_ids, const int32_t* rows_total,
                             int64_t max_rows, uint8_t* perm, float* gsum, uint16_t* sum_parts,
                             int num_sms, cudaStream_t s) {
  if (max_rows == 0) return cudaSuccess;
  if (cudaError_t err = ensure_debug_latch()) return err;
  ep_gather_kernel<<<grid_for(max_rows * 32, 256, num_sms), 256, 0, s>>>(
      codes, T, H, sorted_token_ids, rows_total, perm, gsum, sum_parts);
  return cudaGetLastError();
}

cudaError_t launch_cast_bf16(const float* x, int64_t n, void* out, int num_sms, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 8) return cudaErrorInvalidValue;
  cast_bf16_kernel<<<grid_for(n / 8, 256, num_sms), 256, 0, s>>>(
      x, n / 8, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

cudaError_t launch_inter_quant(const float* h, const uint32_t* row_amax, int64_t A, int64_t I,
                               uint8_t* codes, float* scales, float* gsum, int num_sms,
                               cudaStream_t s, int32_t* int8_row_sum, uint16_t* sum_parts,
                               const int32_t* rows_dev) {
  if (A == 0) return cudaSuccess;
  const int grid = grid_for(A * (I / 16), 256, num_sms);
  if (int8_row_sum) {
    cudaError_t err = cudaMemsetAsync(int8_row_sum, 0, static_cast<size_t>(A) * sizeof(int32_t), s);
    if (err != cudaSuccess) return err;
    if (sum_parts) return cudaErrorInvalidValue;
    inter_quant_kernel<true><<<grid, 256, 0, s>>>(h, row_amax, A, I, codes, scales, nullptr,
                                                  int8_row_sum, nullptr, rows_dev);
  } else {
    inter_quant_kernel<false><<<grid, 256, 0, s>>>(h, row_amax, A, I, codes, scales, gsum,
                                                   nullptr, sum_parts, rows_dev);
  }
  return cudaGetLastError();
}

cudaError_t launch_repack_int4_b200(const int32_t* in, int64_t nwords, int32_t* out, int num_sms,
                                    cudaStream_t s) {
  if (nwords == 0) return cudaSuccess;
  const int grid = grid_for(nwords, 256, num_sms, 16);
  repack_int4_b200_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(in), nwords,
                                               reinterpret_cast<uint32_t*>(out));
  return cudaGetLastError();
}

cudaError_t launch_transpose_scales(const void* in, int64_t E, int64_t rows, int64_t G, void* out,
                                    int num_sms, cudaStream_t s) {
  const int64_t n = E * rows * G;
  if (n == 0) return cudaSuccess;
  const int grid = grid_for(n, 256, num_sms, 16);
  transpose_scales_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(in), E, rows, G,
                                               static_cast<uint16_t*>(out));
  return cudaGetLastError();
}

cudaError_t launch_pack_int4_channel(const void* w, int64_t R, int64_t K, int32_t* packed,
                                     void* scales, int num_sms, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int grid = static_cast<int>(R < cap ? R : cap);
  pack_int4_channel_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), R, K, packed,
                                                static_cast<__nv_bfloat16*>(scales));
  return cudaGetLastError();
}

cudaError_t launch_nibble_row_sum(const int32_t* packed, int64_t R, int64_t words_per_row,
                                  int32_t* sums, int num_sms, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  const int grid = grid_for(R * 32, 256, num_sms, 16);
  nibble_row_sum_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(packed), R,
                                             words_per_row, sums);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* y, const int32_t* row_of, const float* topk_w, int64_t T,
                           int64_t H, int k, void* out, int num_sms, cudaStream_t s,
                           const float* y_shared, float* partial_f32) {
  if (T == 0) return cudaSuccess;
  if (cudaError_t err = ensure_debug_latch()) return err;
  const int grid = grid_for(T * (H / 8), 256, num_sms);
  if (partial_f32)
    combine_kernel<true><<<grid, 256, 0, s>>>(y, row_of, topk_w, T, H, k, nullptr, nullptr,
                                              partial_f32);
  else
    combine_kernel<false><<<grid, 256, 0, s>>>(y, row_of, topk_w, T, H, k, y_shared,
                                               static_cast<__nv_bfloat16*>(out), nullptr);
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8_block(const void* w, int64_t R, int64_t K, uint8_t* codes,
                                   float* scales, cudaStream_t s) {
  if (R == 0 || K == 0) return cudaSuccess;
  if (R / kGroup > 65535) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(K / kGroup), static_cast<unsigned>(R / kGroup));
  quant_fp8_block_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), K, codes,
                                              scales);
  return cudaGetLastError();
}

cudaError_t launch_act_quant_group(const void* x_bf16, const float* x_f32, int64_t T, int64_t H,
                                   uint8_t* codes, float* scales, int num_sms, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if ((x_bf16 == nullptr) == (x_f32 == nullptr)) return cudaErrorInvalidValue;
  const int grid = grid_for(T * (H / 8), 256, num_sms);
  if (x_bf16)
    act_quant_group_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x_bf16), T, H, codes, scales);
  else
    act_quant_group_kernel<float><<<grid, 256, 0, s>>>(x_f32, T, H, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_dense_tables(int32_t* offsets, int32_t* tile_prefix, int64_t T, int tile_n,
                                cudaStream_t s) {
  dense_tables_kernel<<<1, 32, 0, s>>>(offsets, tile_prefix, static_cast<int32_t>(T), tile_n);
  return cudaGetLastError();
}


cudaError_t launch_ep_plan(const int32_t* topk_ids, int64_t T, int k, int E, int n_ranks,
                           int32_t* counts, int32_t* rows, int32_t* pos, cudaStream_t s) {
  if (n_ranks < 1 || n_ranks > kEpMaxRanks) return cudaErrorInvalidValue;
  ep_plan_kernel<<<1, kPlanThreads, 0, s>>>(topk_ids, T, k, E, n_ranks, counts, rows, pos);
  return cudaGetLastError();
}

cudaError_t launch_ep_gather_rows(const uint8_t* codes, const float* scales, const int32_t* ids,
                                  const float* w, int64_t T, int64_t H, int k, const int32_t* rows,
                                  int64_t n_rows, uint8_t* codes_out, float* scales_out,
                                  int32_t* ids_out, float* w_out, int num_sms, cudaStream_t s) {
  if (n_rows == 0) return cudaSuccess;
  if (cudaError_t err = ensure_debug_latch()) return err;
  ep_gather_rows_kernel<<<grid_for(n_rows * 32, 256, num_sms), 256, 0, s>>>(
      codes, scales, ids, w, T, H, k, rows, n_rows, codes_out, scales_out, ids_out, w_out);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine_rows(const float* back, int64_t n_rows, int64_t H,
                                   const int32_t* pos, int64_t T, int n_ranks, void* out,
                                   int num_sms, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (cudaError_t err = ensure_debug_latch()) return err;
  ep_combine_rows_kernel<<<grid_for(T * (H / 8), 256, num_sms), 256, 0, s>>>(
      back, n_rows, H, pos, T, n_ranks, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace w4a8

// Shared device-side helpers of libquoka: element types, the per-call sequence table,
// orderable float keys, warp reductions and the device error word.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "quoka.h"

namespace quoka {

// Per-call description of the batch, passed to kernels by value.
struct SeqTable {
  int batch;
  int max_prefix;
  long long kv_off[QUOKA_MAX_BATCH + 1];
  int prefix[QUOKA_MAX_BATCH];
  int nsel[QUOKA_MAX_BATCH];  // min(budget[b], prefix[b])
};

// Device error word: bit 0 = a bounded wait gave up, bit 2 = an index outside its range,
// bit 3 = a per-query tile's key union exceeded the caller's bound.
__device__ unsigned int g_device_error;

enum : unsigned int { ERR_WAIT_TIMEOUT = 1u, ERR_TMEM_ALLOC = 2u, ERR_BAD_INDEX = 4u, ERR_UNION_CAP = 8u };

__device__ __forceinline__ void flag_error(unsigned int bit) { atomicOr(&g_device_error, bit); }

// ---- element access ------------------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// The two bf16 halves of a 32-bit word (low half = lower address) as floats.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Load N consecutive elements (N * sizeof(T) is 8 or 16 bytes, aligned) as floats.
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T* p, float (&out)[N]);

template <>
__device__ __forceinline__ void load_vec<float, 4>(const float* p, float (&out)[4]) {
  float4 v = __ldg(reinterpret_cast<const float4*>(p));
  out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}
template <>
__device__ __forceinline__ void load_vec<float, 2>(const float* p, float (&out)[2]) {
  float2 v = __ldg(reinterpret_cast<const float2*>(p));
  out[0] = v.x; out[1] = v.y;
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&out)[4]) {
  uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&v.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&v.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  out[0] = fa.x; out[1] = fa.y; out[2] = fb.x; out[3] = fb.y;
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 2>(const __nv_bfloat16* p, float (&out)[2]) {
  unsigned int v = __ldg(reinterpret_cast<const unsigned int*>(p));
  float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v));
  out[0] = f.x; out[1] = f.y;
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&out)[8]) {
  uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
  const unsigned int w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    unsigned int wi = w[i];
    float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wi));
    out[2 * i] = f.x; out[2 * i + 1] = f.y;
  }
}

// ---- orderable keys --------------------------------------------------------------
// Maps a float to a uint32 whose unsigned order equals the float order (-0 and +0
// are first canonicalised to +0 so they compare equal).  NaN is out of contract.
__device__ __forceinline__ uint32_t float_to_ordered(float f) {
  f = f + 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- warp helpers --------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace quoka

// Shared device-side helpers of the LSH attention library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsh_attention_hash.h"

namespace lsh {

// Per-device status word.  Kernels record the first error they detect with
// record_error(); lsh_get_device_status() reads and clears it.
__device__ int g_status = 0;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_status, 0, code); }

// Element loads from bf16 or fp32 storage, widened to fp32.
template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Loads 8 consecutive elements (16 B for bf16, 32 B for fp32) as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* out) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float* out) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

// Stores 8 fp32 values as 8 consecutive elements.
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* in) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float* in) {
  *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(in[4], in[5], in[6], in[7]);
}

// Raw 16-byte copy helpers (row gathers).
__device__ __forceinline__ uint4 ld16(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void st16(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// Hash state of one row: the largest |p_k| with its bucket code, and the
// second largest |p_k|.  Ordering: larger value first, then lower bucket.
struct Top2 {
  float v1;   // largest |p_k|
  int b1;     // bucket of v1: k if p_k >= 0, else k + n_buckets/2
  float v2;   // second largest |p_k| over the other k
};

__device__ __forceinline__ Top2 top2_empty() { return Top2{-INFINITY, 0x7fffffff, -INFINITY}; }

__device__ __forceinline__ bool top2_beats(float va, int ba, float vb, int bb) {
  return va > vb || (va == vb && ba < bb);
}

__device__ __forceinline__ void top2_push(Top2& s, float p, int k, int half) {
  float a = fabsf(p);
  int bk = p >= 0.f ? k : k + half;
  if (top2_beats(a, bk, s.v1, s.b1)) {
    s.v2 = s.v1;
    s.v1 = a;
    s.b1 = bk;
  } else {
    s.v2 = fmaxf(s.v2, a);
  }
}

__device__ __forceinline__ Top2 top2_merge(Top2 a, Top2 b) {
  if (top2_beats(b.v1, b.b1, a.v1, a.b1)) {
    return Top2{b.v1, b.b1, fmaxf(a.v1, b.v2)};
  }
  return Top2{a.v1, a.b1, fmaxf(a.v2, b.v1)};
}

// Near-tie test on the two largest values u1 >= u2 of [p, -p].  With at least
// two columns u2 is the second largest |p_k|; with one column it is -u1.
__device__ __forceinline__ bool top2_near_tie(const Top2& s, float tie_rel) {
  float u1 = s.v1;
  float u2 = fmaxf(s.v2, -u1);
  return (u1 - u2) < tie_rel * fmaxf(u1, 1e-30f);
}

constexpr float kTieRel = 1e-5f;

}  // namespace lsh

// Angular LSH hash, CUDA-core version (exact fp32 FMA; any dtype, any D <= 256).
//
// Ultralytics glossary "Reformer", section "Atencao LSH": bucket = position of
// the largest value of [xR, -xR].  Each CTA takes kHashRows rows and one round;
// thread t owns columns t, t + blockDim, ... of R[round] and keeps, per row, the
// running largest |p_k| (with its bucket code) and the second largest.  The
// per-row states are then merged across the CTA.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kHashRows = 16;
constexpr int kHashThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kHashThreads)
hash_simt_kernel(const T* __restrict__ qk, const T* __restrict__ R, long long nrows, int L, int D,
                 int n_rounds, int half, int32_t* __restrict__ buckets, uint8_t* __restrict__ near_tie) {
  extern __shared__ float xs[];  // [kHashRows][D]
  __shared__ Top2 red[kHashThreads / 32][kHashRows];
  const int round = blockIdx.y;
  const long long row0 = (long long)blockIdx.x * kHashRows;
  const int nr = (int)min((long long)kHashRows, nrows - row0);

  for (int i = threadIdx.x; i < kHashRows * D; i += blockDim.x) {
    int j = i / D, d = i - j * D;
    xs[i] = j < nr ? to_f32(qk[(row0 + j) * D + d]) : 0.f;
  }
  __syncthreads();

  Top2 st[kHashRows];
#pragma unroll
  for (int j = 0; j < kHashRows; ++j) st[j] = top2_empty();

  const T* Rr = R + (size_t)round * D * half;
  for (int k = threadIdx.x; k < half; k += blockDim.x) {
    float acc[kHashRows];
#pragma unroll
    for (int j = 0; j < kHashRows; ++j) acc[j] = 0.f;
    for (int d = 0; d < D; ++d) {
      float r = to_f32(Rr[(size_t)d * half + k]);
#pragma unroll
      for (int j = 0; j < kHashRows; ++j) acc[j] = fmaf(xs[j * D + d], r, acc[j]);
    }
#pragma unroll
    for (int j = 0; j < kHashRows; ++j) top2_push(st[j], acc[j], k, half);
  }

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < kHashRows; ++j) {
    Top2 s = st[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      Top2 o;
      o.v1 = __shfl_xor_sync(0xffffffffu, s.v1, off);
      o.b1 = __shfl_xor_sync(0xffffffffu, s.b1, off);
      o.v2 = __shfl_xor_sync(0xffffffffu, s.v2, off);
      s = top2_merge(s, o);
    }
    if (lane == 0) red[warp][j] = s;
  }
  __syncthreads();
  if (threadIdx.x < nr) {
    const int j = threadIdx.x;
    Top2 s = red[0][j];
    for (int w = 1; w < kHashThreads / 32; ++w) s = top2_merge(s, red[w][j]);
    const long long row = row0 + j;
    const long long bh = row / L;
    const long long l = row - bh * L;
    const size_t o = ((size_t)bh * n_rounds + round) * L + l;
    buckets[o] = s.b1;
    if (near_tie) near_tie[o] = top2_near_tie(s, kTieRel) ? 1 : 0;
  }
}

}  // namespace lsh

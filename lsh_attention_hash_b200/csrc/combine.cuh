// Merge of the hash rounds by their log-sum-exp weights.
//
// twgreatdaily ICLR 2020 Reformer article, section "1 LSH Attention": several
// rounds with different hash functions; each round's output is weighted by
// its share of the total partition function, exp(lse_r - LSE), which gives the
// softmax over the rounds' key sets counted with multiplicity.
//
// Memory-bound: a group of G = D/8 consecutive threads (inside one warp) owns
// one token; each thread streams 8 elements of every round's row (16 B for
// bf16, 32 B for fp32).  With NR (the number of rounds) known at compile time
// all of a thread's loads are issued before any arithmetic, so NR requests per
// thread are in flight together; the NR lse values of the token are loaded by
// the first NR threads of the group and shared by shuffles.
#pragma once

#include "common.cuh"

namespace lsh {

template <typename TI, typename TO, int NR>
__global__ void __launch_bounds__(256)
combine_kernel(const TI* __restrict__ o_r, const float* __restrict__ lse, long long ntok, int L, int D,
               int n_rounds, TO* __restrict__ out, float* __restrict__ lse_out) {
  const int G = D / 8;  // threads per token (1..32; D <= 256)
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long t = gt / G;
  const int piece = (int)(gt - t * G);
  const int lane = threadIdx.x & 31;
  const int leader = lane - piece;  // first lane of this token's group
  const bool live = t < ntok;
  const long long tt = live ? t : 0;
  const long long bh = tt / L, l = tt - bh * L;
  const float* lp = lse + bh * n_rounds * (long long)L + l;
  const TI* op = o_r + (bh * n_rounds * (long long)L + l) * D + piece * 8;
  const long long rstride = (long long)L * D;
  if constexpr (NR > 0) {
    float x[NR][8];
#pragma unroll
    for (int r = 0; r < NR; ++r) load8(op + r * rstride, x[r]);
    float my = (piece < NR && live) ? lp[(long long)piece * L] : 0.f;
    float lv[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) lv[r] = __shfl_sync(0xffffffffu, my, leader + r);
    float mx = lv[0];
#pragma unroll
    for (int r = 1; r < NR; ++r) mx = fmaxf(mx, lv[r]);
    float w[NR], s = 0.f;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      w[r] = expf(lv[r] - mx);
      s += w[r];
    }
    const float inv_s = 1.f / s;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float a = 0.f;
#pragma unroll
      for (int r = 0; r < NR; ++r) a = fmaf(w[r] * inv_s, x[r][e], a);
      acc[e] = a;
    }
    if (!live) return;
    store8(out + t * (long long)D + piece * 8, acc);
    if (lse_out && piece == 0) lse_out[t] = mx + logf(s);
  } else {
    if (!live) return;
    float mx = -INFINITY;
    for (int r = 0; r < n_rounds; ++r) mx = fmaxf(mx, lp[(long long)r * L]);
    float s = 0.f;
    for (int r = 0; r < n_rounds; ++r) s += expf(lp[(long long)r * L] - mx);
    const float inv_s = 1.f / s;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < n_rounds; ++r) {
      const float w = expf(lp[(long long)r * L] - mx) * inv_s;
      float x[8];
      load8(op + r * rstride, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, x[e], acc[e]);
    }
    store8(out + t * (long long)D + piece * 8, acc);
    if (lse_out && piece == 0) lse_out[t] = mx + logf(s);
  }
}

}  // namespace lsh

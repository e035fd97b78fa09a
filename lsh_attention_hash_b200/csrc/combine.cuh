// Merge of the hash rounds by their log-sum-exp weights.
//
// twgreatdaily ICLR 2020 Reformer article, section "1 LSH Attention": several
// rounds with different hash functions; each round's output is weighted by
// its share of the total partition function, exp(lse_r - LSE), which gives the
// softmax over the rounds' key sets counted with multiplicity.
//
// Memory-bound: a group of D/8 threads owns one token and streams its n_rounds
// rows with 16-byte (bf16) / 32-byte (fp32) accesses.
#pragma once

#include "common.cuh"

namespace lsh {

template <typename TI, typename TO>
__global__ void __launch_bounds__(256)
combine_kernel(const TI* __restrict__ o_r, const float* __restrict__ lse, long long ntok, int L, int D,
               int n_rounds, TO* __restrict__ out, float* __restrict__ lse_out) {
  const int G = D / 8;  // threads per token
  const long long t = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / G;
  const int piece = (int)(((long long)blockIdx.x * blockDim.x + threadIdx.x) % G);
  if (t >= ntok) return;
  const long long bh = t / L, l = t - bh * L;
  const float* lp = lse + bh * n_rounds * (long long)L + l;
  float mx = -INFINITY;
  for (int r = 0; r < n_rounds; ++r) mx = fmaxf(mx, lp[(long long)r * L]);
  float s = 0.f;
  for (int r = 0; r < n_rounds; ++r) s += expf(lp[(long long)r * L] - mx);
  const float inv_s = 1.f / s;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int r = 0; r < n_rounds; ++r) {
    const float w = expf(lp[(long long)r * L] - mx) * inv_s;
    float x[8];
    load8(o_r + ((bh * n_rounds + r) * (long long)L + l) * D + piece * 8, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, x[e], acc[e]);
  }
  store8(out + t * (long long)D + piece * 8, acc);
  if (lse_out && piece == 0) lse_out[t] = mx + logf(s);
}

}  // namespace lsh

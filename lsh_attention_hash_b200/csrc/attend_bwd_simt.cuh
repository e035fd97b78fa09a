// Backward of the chunk attention and the round merge, CUDA-core version.
//
// Training through LSH attention recomputes from the stored hash (twgreatdaily
// ICLR 2020 Reformer article, section "1 LSH Attention"; Ultralytics glossary,
// "Atencao LSH"): buckets, sort and masks stay fixed.  With the merged output
// out_i = sum_r sum_j exp(z_ij^r - LSE_i) v_j (the rounds merged by their
// log-sum-exp), the gradient of sum(dout * out) is, per round and admissible
// pair (i, j),
//     p~_ij = exp(z_ij - LSE_i),   dz_ij = p~_ij (dout_i . v_j - dout_i . out_i)
//     dv_j   += p~_ij dout_i
//     dx_i   += scale * dz_ij k_j                  (query role, k_j = x_j / ||x_j||)
//     dk_j   += scale * dz_ij x_i                  (key role)
// and finally dx_j += (dk_j - (dk_j . k_j) k_j) / ||x_j|| (the key normalisation;
// below a length of 1e-12 the clamp is linear: dk_j * 1e12).  z carries the
// union correction -log N_ij when it is on (a constant).
//
// One launch per round.  A CTA owns 32 sorted slots of one chunk k of one
// (b, h) slice: as queries they see chunks k-1 and k (query role), as keys they
// are seen by the queries of chunks k and k+1 (key role).  Both roles add into
// the owned tokens' rows of dqk and dv, which no other CTA of the launch
// touches (perm is a permutation), so there are no atomics and the result is
// deterministic.  Each pair's p~ and dz are computed by both CTAs involved.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kBwdB = 32;      // slots per block (queries or keys)
constexpr int kBwdWarps = 8;   // 4 queries per warp in the pair step

// Shared memory of attend_bwd_simt_kernel, in 4-byte words.
__host__ __device__ inline size_t bwd_smem_words(int D, int n_rounds, int union_count) {
  const size_t DP = (size_t)D + 1;
  return 4 * kBwdB * DP                       // qs, gs, ks, vs
         + 3 * kBwdB * (kBwdB + 1)            // p~, dz, x_i . k_j
         + 2 * (size_t)kBwdB * D              // two accumulators
         + 6 * kBwdB                          // lse, delta, kinv, kproj, ck, pad
         + 7 * kBwdB                          // q_pos, q_slot, q_bk, q_alone, k_pos, k_slot, k_bk
         + (union_count ? 2 * (size_t)n_rounds * kBwdB : 0);
}

template <typename T, typename TO>
__global__ void __launch_bounds__(kBwdWarps * 32)
attend_bwd_simt_kernel(const T* __restrict__ qk, const T* __restrict__ v, const int32_t* __restrict__ perm,
                       const int32_t* __restrict__ buckets, const TO* __restrict__ out,
                       const float* __restrict__ lse, const TO* __restrict__ dout, int L, int D, int n_rounds,
                       int round, int chunk, int self_mask, int causal, int bucket_mask, int union_count,
                       float scale, float* __restrict__ dqk, float* __restrict__ dv) {
  extern __shared__ float sm[];
  const int DP = D + 1;
  float* qs = sm;                          // [32][DP] query rows x_i
  float* gs = qs + kBwdB * DP;             // [32][DP] their dout rows
  float* ks = gs + kBwdB * DP;             // [32][DP] key rows x_j
  float* vs = ks + kBwdB * DP;             // [32][DP] their values
  float* pm = vs + kBwdB * DP;             // [32][33] p~
  float* dz = pm + kBwdB * (kBwdB + 1);    // [32][33] dz
  float* zq = dz + kBwdB * (kBwdB + 1);    // [32][33] x_i . k_j
  float* acc1 = zq + kBwdB * (kBwdB + 1);  // [32][D] query role: dx; key role: dk
  float* acc2 = acc1 + kBwdB * D;          // [32][D] key role: dv
  float* q_lse = acc2 + kBwdB * D;         // [32]
  float* q_delta = q_lse + kBwdB;          // [32] dout_i . out_i
  float* kinv = q_delta + kBwdB;           // [32] 1 / max(||x_j||, 1e-12)
  float* kproj = kinv + kBwdB;             // [32] 1 when ||x_j|| >= 1e-12 (projection term), else 0
  float* ck = kproj + kBwdB;               // [32] key role: dk_j . k_j
  int* q_pos = reinterpret_cast<int*>(ck + 2 * kBwdB);
  int* q_slot = q_pos + kBwdB;
  int* q_bk = q_slot + kBwdB;
  int* q_alone = q_bk + kBwdB;
  int* k_pos = q_alone + kBwdB;
  int* k_slot = k_pos + kBwdB;
  int* k_bk = k_slot + kBwdB;
  int* qbr = k_bk + kBwdB;                 // union: [n_rounds][32]
  int* kbr = qbr + n_rounds * kBwdB;       // union: [n_rounds][32]

  const long long bh = blockIdx.y;
  const long long seg = bh * n_rounds + round;
  const int blocks_per_chunk = (chunk + kBwdB - 1) / kBwdB;
  const int k = blockIdx.x / blocks_per_chunk;
  const int s0 = k * chunk + (blockIdx.x - k * blocks_per_chunk) * kBwdB;  // owned slots [s0, s1)
  const int s1 = min(s0 + kBwdB, (k + 1) * chunk);
  const int n_chunks = L / chunk;
  const int32_t* pseg = perm + seg * L;
  const int32_t* bk_bh = buckets ? buckets + bh * n_rounds * (long long)L : nullptr;
  const int32_t* bk_seg = bk_bh ? bk_bh + (long long)round * L : nullptr;
  const T* qk_bh = qk + bh * (long long)L * D;
  const T* v_bh = v + bh * (long long)L * D;
  const TO* out_bh = out + bh * (long long)L * D;
  const TO* dout_bh = dout + bh * (long long)L * D;
  const float* lse_bh = lse + bh * (long long)L;
  float* dqk_bh = dqk + bh * (long long)L * D;
  float* dv_bh = dv + bh * (long long)L * D;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kThreads = kBwdWarps * 32;

  // Whether the query at sorted slot s has no admissible key but itself (the
  // self slot then stays in); scanned outward from s with an early exit.
  auto alone = [&](int s, int qpos, int qb) -> int {
    const int kq = s / chunk;
    const int w0 = max(kq - 1, 0) * chunk, w1 = (kq + 1) * chunk;
    if (!causal && !bucket_mask) return (w1 - w0) == 1;
    for (int d = 1; d < w1 - w0; ++d) {
#pragma unroll
      for (int side = 0; side < 2; ++side) {
        const int t = side ? s + d : s - d;
        if (t < w0 || t >= w1) continue;
        const int p = pseg[t];
        if ((!causal || p < qpos) && (!bucket_mask || bk_seg[p] == qb)) return 0;
      }
    }
    return 1;
  };

  // Query block: slots [a, a + n).
  auto load_queries = [&](int a, int n) {
    for (int i = tid; i < kBwdB; i += kThreads) {
      const int pos = i < n ? pseg[a + i] : 0;
      q_pos[i] = pos;
      q_slot[i] = a + i;
      q_lse[i] = i < n ? lse_bh[pos] : 0.f;
      const int qb = (bucket_mask && i < n) ? bk_seg[pos] : 0;
      q_bk[i] = qb;
      q_alone[i] = (self_mask && i < n) ? alone(a + i, pos, qb) : 0;  // read only under the self mask
    }
    if (union_count)
      for (int i = tid; i < n_rounds * kBwdB; i += kThreads) {
        const int r = i / kBwdB, j = i - r * kBwdB;
        qbr[i] = j < n ? bk_bh[(long long)r * L + pseg[a + j]] : -1;
      }
    for (int i = tid; i < kBwdB * D; i += kThreads) {
      const int j = i / D, d = i - j * D;
      float x = 0.f, g = 0.f;
      if (j < n) {
        const long long row = (long long)pseg[a + j] * D;
        x = to_f32(qk_bh[row + d]);
        g = to_f32(dout_bh[row + d]);
      }
      qs[j * DP + d] = x;
      gs[j * DP + d] = g;
    }
    for (int i = warp; i < kBwdB; i += kBwdWarps) {  // delta_i = dout_i . out_i
      float acc = 0.f;
      if (i < n) {
        const long long row = (long long)pseg[a + i] * D;
        for (int d = lane; d < D; d += 32) acc = fmaf(to_f32(dout_bh[row + d]), to_f32(out_bh[row + d]), acc);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) q_delta[i] = acc;
    }
  };

  // Key block: slots [a, a + n).
  auto load_keys = [&](int a, int n) {
    for (int i = tid; i < kBwdB; i += kThreads) {
      const int pos = i < n ? pseg[a + i] : 0;
      k_pos[i] = pos;
      k_slot[i] = a + i;
      k_bk[i] = (bucket_mask && i < n) ? bk_seg[pos] : 0;
    }
    if (union_count)
      for (int i = tid; i < n_rounds * kBwdB; i += kThreads) {
        const int r = i / kBwdB, j = i - r * kBwdB;
        kbr[i] = j < n ? bk_bh[(long long)r * L + pseg[a + j]] : -2;
      }
    for (int i = tid; i < kBwdB * D; i += kThreads) {
      const int j = i / D, d = i - j * D;
      float x = 0.f, y = 0.f;
      if (j < n) {
        const long long row = (long long)pseg[a + j] * D;
        x = to_f32(qk_bh[row + d]);
        y = to_f32(v_bh[row + d]);
      }
      ks[j * DP + d] = x;
      vs[j * DP + d] = y;
    }
    __syncthreads();
    for (int j = warp; j < kBwdB; j += kBwdWarps) {
      float ss = 0.f;
      for (int d = lane; d < D; d += 32) ss = fmaf(ks[j * DP + d], ks[j * DP + d], ss);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (lane == 0) {
        const float nrm = sqrtf(ss);
        kinv[j] = 1.f / fmaxf(nrm, 1e-12f);
        kproj[j] = nrm >= 1e-12f ? 1.f : 0.f;
      }
    }
  };

  // p~, dz and x_i . k_j of the loaded query block (nq rows) against the key block (nk).
  auto pairs = [&](int nq, int nk) {
    constexpr int QW = kBwdB / kBwdWarps;
#pragma unroll 1
    for (int a = 0; a < QW; ++a) {
      const int i = warp * QW + a;
      const int j = lane;
      float p = 0.f, g = 0.f, x = 0.f;
      if (i < nq && j < nk) {
        float dot = 0.f, dpv = 0.f;
        for (int d = 0; d < D; ++d) {
          dot = fmaf(qs[i * DP + d], ks[j * DP + d], dot);
          dpv = fmaf(gs[i * DP + d], vs[j * DP + d], dpv);
        }
        x = dot * kinv[j];
        const bool masked = (causal && k_pos[j] > q_pos[i]) || (bucket_mask && k_bk[j] != q_bk[i]) ||
                            (self_mask && k_slot[j] == q_slot[i] && !q_alone[i]);
        if (!masked) {
          float z = scale * x;
          if (union_count) {
            int n_shared = 0;
            for (int r = 0; r < n_rounds; ++r) n_shared += kbr[r * kBwdB + j] == qbr[r * kBwdB + i];
            z -= logf((float)n_shared);
          }
          p = expf(z - q_lse[i]);
          g = p * (dpv - q_delta[i]);
        }
      }
      pm[i * (kBwdB + 1) + j] = p;
      dz[i * (kBwdB + 1) + j] = g;
      zq[i * (kBwdB + 1) + j] = x;
    }
  };

  const int n_own = s1 - s0;

  // ---------------------------------------------------------- query role
  load_queries(s0, n_own);
  for (int i = tid; i < kBwdB * D; i += kThreads) acc1[i] = 0.f;
  {
    const int w0 = max(k - 1, 0) * chunk, w1 = (k + 1) * chunk;
    for (int kb = w0; kb < w1; kb += kBwdB) {
      __syncthreads();  // previous block's readers done
      const int nk = min(kBwdB, w1 - kb);
      load_keys(kb, nk);
      __syncthreads();
      pairs(n_own, nk);
      __syncthreads();
      for (int e = tid; e < kBwdB * D; e += kThreads) {  // dx_i += scale sum_j dz_ij x_j / ||x_j||
        const int i = e / D, d = e - i * D;
        float a = 0.f;
        for (int j = 0; j < nk; ++j) a = fmaf(dz[i * (kBwdB + 1) + j], ks[j * DP + d] * kinv[j], a);
        acc1[e] = fmaf(scale, a, acc1[e]);
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < n_own * D; e += kThreads) {
    const int i = e / D, d = e - i * D;
    dqk_bh[(long long)q_pos[i] * D + d] += acc1[e];
  }
  __syncthreads();

  // ---------------------------------------------------------- key role
  load_keys(s0, n_own);  // ends with the key lengths; a barrier follows below
  for (int i = tid; i < kBwdB * D; i += kThreads) {
    acc1[i] = 0.f;
    acc2[i] = 0.f;
  }
  for (int i = tid; i < kBwdB; i += kThreads) ck[i] = 0.f;
  {
    const int q0 = k * chunk, q1 = min(k + 2, n_chunks) * chunk;  // queries of chunks k and k+1
    for (int qb = q0; qb < q1; qb += kBwdB) {
      __syncthreads();
      const int nq = min(kBwdB, q1 - qb);
      load_queries(qb, nq);
      __syncthreads();
      pairs(nq, n_own);
      __syncthreads();
      for (int j = warp; j < kBwdB; j += kBwdWarps) {  // dk_j . k_j += scale sum_i dz_ij (x_i . k_j)
        float a = lane < nq ? dz[lane * (kBwdB + 1) + j] * zq[lane * (kBwdB + 1) + j] : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        if (lane == 0) ck[j] = fmaf(scale, a, ck[j]);
      }
      for (int e = tid; e < kBwdB * D; e += kThreads) {
        const int j = e / D, d = e - j * D;
        float a = 0.f, b = 0.f;
        for (int i = 0; i < nq; ++i) {
          a = fmaf(dz[i * (kBwdB + 1) + j], qs[i * DP + d], a);
          b = fmaf(pm[i * (kBwdB + 1) + j], gs[i * DP + d], b);
        }
        acc1[e] = fmaf(scale, a, acc1[e]);
        acc2[e] += b;
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < n_own * D; e += kThreads) {
    const int j = e / D, d = e - j * D;
    const float khat = ks[j * DP + d] * kinv[j];
    const long long o = (long long)k_pos[j] * D + d;
    dqk_bh[o] += (acc1[e] - kproj[j] * ck[j] * khat) * kinv[j];
    dv_bh[o] += acc2[e];
  }
}

}  // namespace lsh

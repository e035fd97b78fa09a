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
// The pair step reads 16-byte pieces of the staged rows (one key piece serves
// four queries); the gradients of a warp's four rows stay in registers.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kBwdB = 32;      // slots per block (queries or keys)
constexpr int kBwdWarps = 8;   // 4 queries (pair step, query role) or 4 keys (key role) per warp

// Row stride of the staged rows: D + 4 words keeps every row 16-byte aligned and,
// as D % 8 == 0, makes it an odd multiple of 4 words, so eight lanes reading
// float4s of eight different rows hit 32 different banks.
__host__ __device__ inline int bwd_row_stride(int D) { return D + 4; }

// Shared memory of attend_bwd_simt_kernel, in 4-byte words.
__host__ __device__ inline size_t bwd_smem_words(int D, int n_rounds, int union_count) {
  return 4 * (size_t)kBwdB * bwd_row_stride(D)  // qs, gs, ks, vs
         + 3 * kBwdB * (kBwdB + 1)              // p~, dz, x_i . k_j
         + 6 * kBwdB                            // lse, delta, kinv, kproj, ck, pad
         + 7 * kBwdB                            // q_pos, q_slot, q_bk, q_alone, k_pos, k_slot, k_bk
         + (union_count ? 2 * (size_t)n_rounds * kBwdB : 0);
}

// MDL: columns per lane (D <= 32 * MDL); 4 (D <= 128) leaves room for two CTAs per SM.
template <typename T, typename TO, int MDL>
__global__ void __launch_bounds__(kBwdWarps * 32, MDL <= 4 ? 2 : 1)
attend_bwd_simt_kernel(const T* __restrict__ qk, const T* __restrict__ v, const int32_t* __restrict__ perm,
                       const int32_t* __restrict__ buckets, const TO* __restrict__ out,
                       const float* __restrict__ lse, const TO* __restrict__ dout, int L, int D, int n_rounds,
                       int round, int chunk, int self_mask, int causal, int bucket_mask, int union_count,
                       float scale, float* __restrict__ dqk, float* __restrict__ dv) {
  extern __shared__ __align__(16) float bwd_sm[];
  const int DS = bwd_row_stride(D);
  float* qs = bwd_sm;                        // [32][DS] query rows x_i
  float* gs = qs + kBwdB * DS;             // [32][DS] their dout rows
  float* ks = gs + kBwdB * DS;             // [32][DS] key rows x_j
  float* vs = ks + kBwdB * DS;             // [32][DS] their values
  float* pm = vs + kBwdB * DS;             // [32][33] p~
  float* dz = pm + kBwdB * (kBwdB + 1);    // [32][33] dz
  float* zq = dz + kBwdB * (kBwdB + 1);    // [32][33] x_i . k_j
  float* q_lse = zq + kBwdB * (kBwdB + 1); // [32]
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
  const int r0 = warp * 4;                 // this warp's 4 rows (queries or keys) of a block
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
      qs[j * DS + d] = x;
      gs[j * DS + d] = g;
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

  // Key block: slots [a, a + n); ends with a barrier and the key lengths.
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
      ks[j * DS + d] = x;
      vs[j * DS + d] = y;
    }
    __syncthreads();
    for (int j = warp; j < kBwdB; j += kBwdWarps) {
      float ss = 0.f;
      for (int d = lane; d < D; d += 32) ss = fmaf(ks[j * DS + d], ks[j * DS + d], ss);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (lane == 0) {
        const float nrm = sqrtf(ss);
        kinv[j] = 1.f / fmaxf(nrm, 1e-12f);
        kproj[j] = nrm >= 1e-12f ? 1.f : 0.f;
      }
    }
  };

  // p~, dz and x_i . k_j of the loaded query block (nq rows) against the key
  // block (nk): the warp takes queries r0..r0+3, lane j takes key j; each
  // 16-byte load of a key (and its value) row serves four queries.
  auto pairs = [&](int nq, int nk) {
    const int j = lane;
    float dot[4] = {0.f, 0.f, 0.f, 0.f}, dpv[4] = {0.f, 0.f, 0.f, 0.f};
    if (j < nk) {
      for (int d = 0; d < D; d += 4) {
        const float4 kk = *reinterpret_cast<const float4*>(ks + j * DS + d);
        const float4 vv = *reinterpret_cast<const float4*>(vs + j * DS + d);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const float4 q = *reinterpret_cast<const float4*>(qs + (r0 + a) * DS + d);
          const float4 g = *reinterpret_cast<const float4*>(gs + (r0 + a) * DS + d);
          dot[a] = fmaf(q.x, kk.x, fmaf(q.y, kk.y, fmaf(q.z, kk.z, fmaf(q.w, kk.w, dot[a]))));
          dpv[a] = fmaf(g.x, vv.x, fmaf(g.y, vv.y, fmaf(g.z, vv.z, fmaf(g.w, vv.w, dpv[a]))));
        }
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = r0 + a;
      float p = 0.f, g = 0.f, x = 0.f;
      if (i < nq && j < nk) {
        x = dot[a] * kinv[j];
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
          g = p * (dpv[a] - q_delta[i]);
        }
      }
      pm[i * (kBwdB + 1) + j] = p;
      dz[i * (kBwdB + 1) + j] = g;
      zq[i * (kBwdB + 1) + j] = x;
    }
  };

  const int n_own = s1 - s0;
  const int DL = (D + 31) / 32;

  // ---------------------------------------------------------- query role
  // dx_i = scale sum_j dz_ij x_j / ||x_j||, kept in registers: warp rows r0..r0+3,
  // lane columns lane + 32 e
  {
    float aq[4][MDL];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int e = 0; e < MDL; ++e) aq[a][e] = 0.f;
    load_queries(s0, n_own);
    const int w0 = max(k - 1, 0) * chunk, w1 = (k + 1) * chunk;
    for (int kb = w0; kb < w1; kb += kBwdB) {
      __syncthreads();  // previous block's readers done
      const int nk = min(kBwdB, w1 - kb);
      load_keys(kb, nk);
      __syncthreads();
      pairs(n_own, nk);
      __syncthreads();
      for (int j = 0; j < nk; ++j) {
        const float kj = scale * kinv[j];
        float w[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) w[a] = dz[(r0 + a) * (kBwdB + 1) + j] * kj;
#pragma unroll
        for (int e = 0; e < MDL; ++e) {
          const int d = lane + 32 * e;
          if (e < DL && d < D) {
            const float kd = ks[j * DS + d];
#pragma unroll
            for (int a = 0; a < 4; ++a) aq[a][e] = fmaf(w[a], kd, aq[a][e]);
          }
        }
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      if (r0 + a >= n_own) continue;
      float* dst = dqk_bh + (long long)q_pos[r0 + a] * D;
#pragma unroll
      for (int e = 0; e < MDL; ++e) {
        const int d = lane + 32 * e;
        if (e < DL && d < D) dst[d] += aq[a][e];
      }
    }
  }
  __syncthreads();  // the query role's adds land before the key role adds to the same rows

  // ---------------------------------------------------------- key role
  // dk_j = scale sum_i dz_ij x_i and dv_j = sum_i p~_ij dout_i in registers: warp keys
  // r0..r0+3, lane columns lane + 32 e
  {
    float ak[4][MDL], av[4][MDL];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int e = 0; e < MDL; ++e) {
        ak[a][e] = 0.f;
        av[a][e] = 0.f;
      }
    load_keys(s0, n_own);
    for (int i = tid; i < kBwdB; i += kThreads) ck[i] = 0.f;
    const int q0 = k * chunk, q1 = min(k + 2, n_chunks) * chunk;  // queries of chunks k and k+1
    for (int qb = q0; qb < q1; qb += kBwdB) {
      __syncthreads();
      const int nq = min(kBwdB, q1 - qb);
      load_queries(qb, nq);
      __syncthreads();
      pairs(nq, n_own);
      __syncthreads();
      for (int j = warp; j < kBwdB; j += kBwdWarps) {  // dk_j . k_j += scale sum_i dz_ij (x_i . k_j)
        float c = lane < nq ? dz[lane * (kBwdB + 1) + j] * zq[lane * (kBwdB + 1) + j] : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
        if (lane == 0) ck[j] = fmaf(scale, c, ck[j]);
      }
      for (int i = 0; i < nq; ++i) {
        float wz[4], wp[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          wz[a] = dz[i * (kBwdB + 1) + r0 + a];
          wp[a] = pm[i * (kBwdB + 1) + r0 + a];
        }
#pragma unroll
        for (int e = 0; e < MDL; ++e) {
          const int d = lane + 32 * e;
          if (e < DL && d < D) {
            const float xd = qs[i * DS + d], gd = gs[i * DS + d];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              ak[a][e] = fmaf(wz[a], xd, ak[a][e]);
              av[a][e] = fmaf(wp[a], gd, av[a][e]);
            }
          }
        }
      }
    }
    __syncthreads();  // ck complete
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int j = r0 + a;
      if (j >= n_own) continue;
      const long long row = (long long)k_pos[j] * D;
#pragma unroll
      for (int e = 0; e < MDL; ++e) {
        const int d = lane + 32 * e;
        if (e < DL && d < D) {
          const float khat = ks[j * DS + d] * kinv[j];
          dqk_bh[row + d] += (scale * ak[a][e] - kproj[j] * ck[j] * khat) * kinv[j];
          dv_bh[row + d] += av[a][e];
        }
      }
    }
  }
}

}  // namespace lsh

// Chunk attention, CUDA-core version (fp32 arithmetic; any dtype, chunk, D <= 256).
//
// twgreatdaily ICLR 2020 Reformer article, section "1 LSH Attention": the
// output of query i is the sum over its admissible keys of exp(logit) v_j
// divided by the partition function; with Q = K the keys are length-normalised;
// after sorting, chunk k looks back one chunk (no wrap-around for chunk 0).
// A query does not see its own slot unless that slot is its only key.
// Causal variant (the pages' character-level language model): a key whose
// original position is after the query's is not admissible; a query left with
// no key but itself sees only itself (output v_self, lse = scale * ||q||).
// Bucket-equality variant (same article, same section: the admissible set is the
// query's own bucket, batched by chunks): a key of the window in another bucket
// than the query's in this round is not admissible.  Union correction (same
// section, several rounds): each admissible logit is lowered by log N, N = the
// number of rounds in which query and key share a bucket, so that the rounds
// merged by their log-sum-exp count each shared key once.
//
// One CTA takes up to 32 queries of one chunk of one (b, h, round) segment and
// streams the chunk's window (chunks k-1 and k) in blocks of 32 keys, keeping
// an online softmax per query.  Rows are gathered through perm (or read from
// pre-sorted copies).  Results are written at the original position perm[s].
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kAttQ = 32;     // queries per CTA
constexpr int kAttK = 32;     // keys per block
constexpr int kAttWarps = 8;  // 4 queries per warp
constexpr int kAttMaxDL = 8;  // D / 32 values per lane, D <= 256

template <typename T, typename TO>
__global__ void __launch_bounds__(kAttWarps * 32)
attend_simt_kernel(const T* __restrict__ qk, const T* __restrict__ v, const int32_t* __restrict__ perm,
                   const int32_t* __restrict__ buckets, const T* __restrict__ qk_sorted,
                   const T* __restrict__ v_sorted, int L, int D, int n_rounds, int chunk, int self_mask,
                   int causal, int bucket_mask, int union_count, float scale, TO* __restrict__ out,
                   float* __restrict__ lse) {
  extern __shared__ float sm[];
  const int DP = D + 1;                 // padded row pitch (conflict-free column reads)
  float* qs = sm;                       // [kAttQ][DP]
  float* ks = qs + kAttQ * DP;          // [kAttK][DP]
  float* vs = ks + kAttK * DP;          // [kAttK][D]
  float* kinv = vs + kAttK * D;         // [kAttK]
  int* kbr = reinterpret_cast<int*>(kinv + kAttK);  // union only: [n_rounds][kAttK] key buckets
  int* qbr = kbr + n_rounds * kAttK;                // union only: [n_rounds][kAttQ] query buckets

  const long long seg = blockIdx.y;     // (bh, round)
  const long long bh = seg / n_rounds;
  const int qb_per_chunk = (chunk + kAttQ - 1) / kAttQ;
  const int k = blockIdx.x / qb_per_chunk;
  const int q0 = k * chunk + (blockIdx.x - k * qb_per_chunk) * kAttQ;
  const int q1 = min(q0 + kAttQ, (k + 1) * chunk);
  const int w0 = max(k - 1, 0) * chunk, w1 = (k + 1) * chunk;
  const bool only_self_possible = (w1 - w0) == 1;
  const int32_t* pseg = perm + seg * L;
  const int r_seg = (int)(seg - bh * n_rounds);                       // this segment's round
  const int32_t* bk_bh = buckets ? buckets + bh * n_rounds * (long long)L : nullptr;  // [n_rounds][L]
  const int32_t* bk_seg = bk_bh ? bk_bh + (long long)r_seg * L : nullptr;
  // the self slot is dropped while other keys may remain; it comes back below when none does
  const bool self_fallback = causal || bucket_mask || !only_self_possible;
  const T* qk_bh = qk + bh * (long long)L * D;
  const T* v_bh = v + bh * (long long)L * D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  auto row_qk = [&](int slot) -> const T* {
    return qk_sorted ? qk_sorted + (seg * L + slot) * (long long)D : qk_bh + (long long)pseg[slot] * D;
  };
  auto row_v = [&](int slot) -> const T* {
    return v_sorted ? v_sorted + (seg * L + slot) * (long long)D : v_bh + (long long)pseg[slot] * D;
  };

  for (int i = threadIdx.x; i < kAttQ * D; i += blockDim.x) {
    int j = i / D, d = i - j * D;
    qs[j * DP + d] = (q0 + j < q1) ? to_f32(row_qk(q0 + j)[d]) : 0.f;
  }
  if (union_count) {
    for (int i = threadIdx.x; i < n_rounds * kAttQ; i += blockDim.x) {
      const int r = i / kAttQ, j = i - r * kAttQ;
      qbr[i] = (q0 + j < q1) ? bk_bh[(long long)r * L + pseg[q0 + j]] : -1;
    }
  }

  const int QW = kAttQ / kAttWarps;
  float m[QW], l[QW], o[QW][kAttMaxDL];
#pragma unroll
  for (int a = 0; a < QW; ++a) {
    m[a] = -INFINITY;
    l[a] = 0.f;
#pragma unroll
    for (int e = 0; e < kAttMaxDL; ++e) o[a][e] = 0.f;
  }
  const int DL = (D + 31) / 32;

  for (int kb = w0; kb < w1; kb += kAttK) {
    __syncthreads();
    const int nk = min(kAttK, w1 - kb);
    for (int i = threadIdx.x; i < kAttK * D; i += blockDim.x) {
      int j = i / D, d = i - j * D;
      float x = 0.f, y = 0.f;
      if (j < nk) {
        x = to_f32(row_qk(kb + j)[d]);
        y = to_f32(row_v(kb + j)[d]);
      }
      ks[j * DP + d] = x;
      vs[j * D + d] = y;
    }
    if (union_count) {
      for (int i = threadIdx.x; i < n_rounds * kAttK; i += blockDim.x) {
        const int r = i / kAttK, j = i - r * kAttK;
        kbr[i] = (j < nk) ? bk_bh[(long long)r * L + pseg[kb + j]] : -2;
      }
    }
    __syncthreads();
    if (warp < kAttK / 8) {  // 4 warps x 8 rows: inverse key lengths
      for (int j = warp * 8; j < warp * 8 + 8; ++j) {
        float ss = 0.f;
        for (int d = lane; d < D; d += 32) ss = fmaf(ks[j * DP + d], ks[j * DP + d], ss);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (lane == 0) kinv[j] = 1.f / fmaxf(sqrtf(ss), 1e-12f);
      }
    }
    __syncthreads();
    const int kpos = ((causal || bucket_mask) && lane < nk) ? pseg[kb + lane] : 0;  // lane's key position
    const int kbk = (bucket_mask && lane < nk) ? bk_seg[kpos] : 0;                    // and its bucket
#pragma unroll
    for (int a = 0; a < QW; ++a) {
      const int qi = warp * QW + a;
      const int qslot = q0 + qi;
      if (qslot >= q1) continue;  // warp-uniform
      // lane t scores key kb + t
      float dotv = 0.f;
      for (int d = 0; d < D; ++d) dotv = fmaf(qs[qi * DP + d], ks[lane * DP + d], dotv);
      float logit = dotv * kinv[lane] * scale;
      const int kslot = kb + lane;
      const int qpos = pseg[qslot];
      // self is dropped here while other keys may remain (plain window: unless it is the query
      // alone); a causal or bucket-masked query left with no key falls back to itself below
      const bool masked = lane >= nk || (self_mask && kslot == qslot && self_fallback) ||
                          (causal && kpos > qpos) || (bucket_mask && kbk != bk_seg[qpos]);
      if (masked) {
        logit = -INFINITY;
      } else if (union_count) {
        int n_shared = 0;
        for (int r = 0; r < n_rounds; ++r) n_shared += kbr[r * kAttK + lane] == qbr[r * kAttQ + qi];
        logit -= logf((float)n_shared);  // >= 1: the key passed this round's bucket test
      }
      float bm = logit;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
      const float mn = fmaxf(m[a], bm);
      if (mn == -INFINITY) continue;  // every key of this block masked (warp-uniform)
      const float alpha = expf(m[a] - mn);
      const float p = expf(logit - mn);
      float ps = p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[a] = l[a] * alpha + ps;
      m[a] = mn;
#pragma unroll
      for (int e = 0; e < kAttMaxDL; ++e) o[a][e] *= alpha;
      for (int t = 0; t < nk; ++t) {
        const float pt = __shfl_sync(0xffffffffu, p, t);
#pragma unroll
        for (int e = 0; e < kAttMaxDL; ++e)
          if (e < DL && lane + 32 * e < D) o[a][e] = fmaf(pt, vs[t * D + lane + 32 * e], o[a][e]);
      }
    }
  }

#pragma unroll
  for (int a = 0; a < QW; ++a) {
    const int qi = warp * QW + a;
    const int qslot = q0 + qi;
    if (qslot >= q1) continue;
    const long long pos = pseg[qslot];
    TO* dst = out + (seg * L + pos) * (long long)D;
    if (m[a] == -INFINITY) {  // no admissible key but itself: the query sees only itself
      float ss = 0.f;
      for (int d = lane; d < D; d += 32) ss = fmaf(qs[qi * DP + d], qs[qi * DP + d], ss);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const T* vrow = row_v(qslot);
      for (int d = lane; d < D; d += 32) dst[d] = from_f32<TO>(to_f32(vrow[d]));
      // its logit: scale * ||q|| (q . q / ||q||), less log n_rounds under the union correction
      if (lane == 0) lse[seg * L + pos] = sqrtf(ss) * scale - (union_count ? logf((float)n_rounds) : 0.f);
      continue;
    }
    const float inv_l = 1.f / l[a];
#pragma unroll
    for (int e = 0; e < kAttMaxDL; ++e)
      if (e < DL && lane + 32 * e < D) dst[lane + 32 * e] = from_f32<TO>(o[a][e] * inv_l);
    if (lane == 0) lse[seg * L + pos] = m[a] + logf(l[a]);
  }
}

}  // namespace lsh

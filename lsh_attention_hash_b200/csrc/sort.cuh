// Stable bucket sort of each (b, h, round) segment, and the sorted-row gather.
//
// twgreatdaily ICLR 2020 Reformer article, section "1 LSH Attention": tokens
// are ordered first by bucket and then by position inside the bucket.  Since
// positions already ascend within a segment, this is one stable counting sort
// on the bucket id:
//   1. count:   per (segment, tile of T positions) histogram of bucket ids,
//               stored bucket-major: cnt[seg][bucket][tile];
//   2. scan:    exclusive prefix sum over each segment's cnt array, which makes
//               cnt[seg][b][t] the first sorted slot of bucket b's elements in
//               tile t;
//   3. scatter: one warp walks its tile in position order and places every
//               element at cnt + (number of equal ids before it), ranking equal
//               ids inside a group of 32 with a warp match.
// No step waits on another CTA, so there is no inter-CTA spin.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kSortMinTile = 4096;
constexpr int kSortSmemBuckets = 16384;  // counters kept in shared memory up to this many buckets

__host__ __device__ inline int sort_tile(int n_buckets) {
  return n_buckets > kSortMinTile ? n_buckets : kSortMinTile;
}

__host__ inline size_t sort_ws_elems(long long segs, int L, int n_buckets) {
  const int T = sort_tile(n_buckets);
  const long long nt = (L + T - 1) / T;
  return (size_t)segs * n_buckets * nt;
}

// 1. histogram of one tile.
__global__ void __launch_bounds__(256)
sort_count_kernel(const int32_t* __restrict__ buckets, int L, int n_buckets, int T,
                  uint32_t* __restrict__ cnt) {
  extern __shared__ uint32_t hist[];
  // segments on grid.x (up to 2^31 - 1 of them), tiles on grid.y (at most L / 4096 <= 4096)
  const int tile = blockIdx.y, nt = gridDim.y;
  const long long seg = blockIdx.x;
  const bool in_smem = n_buckets <= kSortSmemBuckets;
  uint32_t* gcnt = cnt + (size_t)seg * n_buckets * nt;
  if (in_smem) {
    for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) hist[b] = 0;
    __syncthreads();
  }
  const int32_t* src = buckets + (size_t)seg * L;
  const int lo = tile * T, hi = min(L, lo + T);
  for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    int b = src[i];
    if ((unsigned)b >= (unsigned)n_buckets) {
      record_error(LSH_ERR_INVALID_ARG);
      continue;
    }
    if (in_smem) atomicAdd(&hist[b], 1u);
    else atomicAdd(&gcnt[(size_t)b * nt + tile], 1u);
  }
  if (in_smem) {
    __syncthreads();
    for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) gcnt[(size_t)b * nt + tile] = hist[b];
  }
}

// 2. exclusive scan of one segment's n = n_buckets * nt counters (1024 threads,
// 4 counters per thread per step, carried across steps).
__global__ void __launch_bounds__(1024) sort_scan_kernel(uint32_t* __restrict__ cnt, long long n) {
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t carry_s;
  uint32_t* a = cnt + (size_t)blockIdx.x * n;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (long long base = 0; base < n; base += 4 * 1024) {
    const long long i0 = base + 4ll * threadIdx.x;
    uint32_t x[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) x[q] = (i0 + q < n) ? a[i0 + q] : 0u;
    uint32_t local = x[0] + x[1] + x[2] + x[3];
    uint32_t incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      uint32_t w = warp_sums[lane];
      uint32_t wi = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, wi, off);
        if (lane >= off) wi += y;
      }
      warp_sums[lane] = wi - w;  // exclusive prefix of warp totals
    }
    __syncthreads();
    const uint32_t carry = carry_s;
    uint32_t run = carry + warp_sums[warp] + incl - local;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (i0 + q < n) a[i0 + q] = run;
      run += x[q];
    }
    __syncthreads();
    if (threadIdx.x == 1023) carry_s = run;
    __syncthreads();
  }
}

// 3. stable scatter of one tile by one warp.
__global__ void __launch_bounds__(32)
sort_scatter_kernel(const int32_t* __restrict__ buckets, int L, int n_buckets, int T,
                    uint32_t* __restrict__ cnt, int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  extern __shared__ uint32_t run[];
  const int tile = blockIdx.y, nt = gridDim.y;
  const long long seg = blockIdx.x;
  const int lane = threadIdx.x;
  const bool in_smem = n_buckets <= kSortSmemBuckets;
  uint32_t* gcnt = cnt + (size_t)seg * n_buckets * nt;
  if (in_smem) {
    for (int b = lane; b < n_buckets; b += 32) run[b] = gcnt[(size_t)b * nt + tile];
    __syncwarp();
  }
  const int32_t* src = buckets + (size_t)seg * L;
  int32_t* dst = perm + (size_t)seg * L;
  int32_t* idst = inv ? inv + (size_t)seg * L : nullptr;
  const int lo = tile * T, hi = min(L, lo + T);
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    int b = i < hi ? src[i] : -1;
    const bool valid = (unsigned)b < (unsigned)n_buckets;
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    unsigned peers = 0;
    uint32_t slot = 0;
    if (valid) {
      peers = __match_any_sync(vmask, b);
      uint32_t* c = in_smem ? &run[b] : &gcnt[(size_t)b * nt + tile];
      slot = *c + __popc(peers & lt_mask);
    }
    __syncwarp();
    if (valid && (peers & lt_mask) == 0) {
      uint32_t* c = in_smem ? &run[b] : &gcnt[(size_t)b * nt + tile];
      *c += __popc(peers);
    }
    __syncwarp();
    if (valid) {
      dst[slot] = i;
      if (idst) idst[i] = (int32_t)slot;
    }
  }
}

// Whole-segment sort in one CTA (L <= 65536, n_buckets <= 1024): each of the
// 32 warps counts a contiguous range of the segment into its own histogram, the
// CTA turns the (bucket, warp) counts into exclusive offsets (bucket-major, so
// warp ranges stay in position order inside a bucket), and each warp then
// places its range in order with the warp-match ranking of
// sort_scatter_kernel.  Counts, offsets and sorted slots are all below 65536,
// so the histograms are uint16 (two buckets per 32-bit word for the counting
// atomics; a warp counts at most 2048 ids, so no carry crosses into the
// neighbour).  The permutation is built in shared memory as uint16 (positions
// < 65536) and written out with coalesced stores; the inverse is written
// directly (its writes are already in position order).
constexpr int kSegWarps = 32;
constexpr int kSegMaxL = 65536;
constexpr int kSegMaxBuckets = 1024;

__host__ __device__ inline size_t sort_segment_smem(int L, int n_buckets) {
  return (size_t)kSegWarps * ((n_buckets + 1) & ~1) * 2  // per-warp histograms / offsets, uint16
         + (size_t)kSegMaxBuckets * 4           // bucket totals / bases
         + 48 * 4                               // warp sums of the scan, count of invalid ids
         + (((size_t)L * 2 + 15) & ~(size_t)15);  // the permutation, uint16
}

__global__ void __launch_bounds__(kSegWarps * 32)
sort_segment_kernel(const int32_t* __restrict__ buckets, int L, int n_buckets, int32_t* __restrict__ perm,
                    int32_t* __restrict__ inv) {
  extern __shared__ uint32_t sm_u32[];
  const int nbp = (n_buckets + 1) & ~1;             // row pitch (even: rows start on a 32-bit word)
  uint16_t* hist = reinterpret_cast<uint16_t*>(sm_u32);  // [kSegWarps][nbp]
  uint32_t* tot = sm_u32 + kSegWarps * nbp / 2;     // [n_buckets]
  uint32_t* ws = tot + kSegMaxBuckets;              // [32] warp sums, [32] invalid ids
  uint16_t* pm = reinterpret_cast<uint16_t*>(ws + 48);  // [L] sorted slot -> position
  const long long seg = blockIdx.x;
  const int32_t* src = buckets + seg * L;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per_warp = (((L + kSegWarps - 1) / kSegWarps) + 31) & ~31;
  const int lo = min(L, warp * per_warp), hi = min(L, lo + per_warp);

  for (int i = threadIdx.x; i < kSegWarps * nbp / 2; i += blockDim.x) sm_u32[i] = 0;
  if (threadIdx.x == 0) ws[32] = 0;
  __syncthreads();
  // 1. per-warp counts of a contiguous range (out-of-range ids are skipped)
  uint16_t* my = hist + warp * nbp;
  uint32_t* my_words = sm_u32 + warp * nbp / 2;
  for (int base = lo; base < hi; base += 128) {
    int bq[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = base + 32 * k + lane;
      bq[k] = i < hi ? src[i] : 0x7fffffff;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (base + 32 * k + lane >= hi) continue;
      const int b = bq[k];
      if ((unsigned)b >= (unsigned)n_buckets) {
        record_error(LSH_ERR_INVALID_ARG);
        atomicAdd(&ws[32], 1u);
      } else {
        atomicAdd(&my_words[b >> 1], 1u << (16 * (b & 1)));
      }
    }
  }
  __syncthreads();
  // 2a. within each bucket, exclusive offsets over the warps (in warp = position order)
  for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) {
    uint32_t run = 0;
    for (int w = 0; w < kSegWarps; ++w) {
      const uint32_t c = hist[w * nbp + b];
      hist[w * nbp + b] = (uint16_t)run;  // < 65536: at most L - (this warp's count)
      run += c;
    }
    tot[b] = run;
  }
  __syncthreads();
  // 2b. exclusive scan of the bucket totals (one bucket per thread)
  {
    const int b0 = threadIdx.x;
    const uint32_t local = b0 < n_buckets ? tot[b0] : 0u;
    uint32_t incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) ws[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t w = lane < kSegWarps ? ws[lane] : 0u;
      uint32_t wi = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, wi, off);
        if (lane >= off) wi += y;
      }
      if (lane < kSegWarps) ws[lane] = wi - w;
    }
    __syncthreads();
    const uint32_t excl = ws[warp] + incl - local;
    if (b0 < n_buckets) tot[b0] = excl;
  }
  __syncthreads();
  // 2c. first sorted slot of (bucket, warp)
  for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) {
    const uint32_t base = tot[b];
    for (int w = 0; w < kSegWarps; ++w) hist[w * nbp + b] = (uint16_t)(hist[w * nbp + b] + base);  // a slot < L
  }
  __syncthreads();
  // 3. stable placement of the warp's range (ids re-read, now from L2, four groups
  //    of 32 at a time so that the loads overlap)
  int32_t* idst = inv ? inv + seg * L : nullptr;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 128) {
    int bq[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = base + 32 * k + lane;
      bq[k] = i < hi ? src[i] : -1;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = base + 32 * k + lane;
      const int b = bq[k];
      const bool valid = (unsigned)b < (unsigned)n_buckets;
      const unsigned vmask = __ballot_sync(0xffffffffu, valid);
      unsigned peers = 0;
      uint32_t slot = 0;
      if (valid) {
        peers = __match_any_sync(vmask, b);
        slot = my[b] + __popc(peers & lt_mask);
      }
      __syncwarp();
      if (valid && (peers & lt_mask) == 0) my[b] = (uint16_t)(my[b] + __popc(peers));
      __syncwarp();
      if (valid) {
        pm[slot] = (uint16_t)i;
        if (idst) idst[i] = (int32_t)slot;
      }
    }
  }
  __syncthreads();
  // 4. coalesced write of the permutation: the valid ids fill slots [0, n_valid);
  //    slots past it (left by out-of-range ids) stay as they were.
  const uint32_t n_valid = (uint32_t)L - ws[32];
  int32_t* dst = perm + seg * L;
  for (int s = threadIdx.x; s < L; s += blockDim.x)
    if ((uint32_t)s < n_valid) dst[s] = pm[s];
}

// Gather of sorted rows: dst[seg][s][:] = src[bh][perm[seg][s]][:], 16 B per thread.
__global__ void gather_rows_kernel(const uint8_t* __restrict__ src, const int32_t* __restrict__ perm,
                                   long long n_rows, int L, int n_rounds, int row_bytes,
                                   uint8_t* __restrict__ dst) {
  const int per_row = row_bytes / 16;
  const long long total = n_rows * per_row;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long row = t / per_row;          // row of the [B, H, n_rounds, L] index space
    const int piece = (int)(t - row * per_row);
    const long long seg = row / L;              // (bh, round)
    const long long bh = seg / n_rounds;
    const int p = perm[row];
    const uint8_t* s = src + ((size_t)bh * L + p) * row_bytes + piece * 16;
    st16(dst + (size_t)row * row_bytes + piece * 16, ld16(s));
  }
}

}  // namespace lsh

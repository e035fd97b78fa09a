// Stable bucket sort of each (b, h, round) segment, and the sorted-row gather.
//
// twgreatdaily ICLR 2020 Reformer article, section "1 LSH Attention": tokens
// are ordered first by bucket and then by position inside the bucket.  Since
// positions already ascend within a segment, this is a stable sort on the
// bucket id alone.  Segments of at most 65536 positions and 1024 buckets are
// sorted by one CTA each (sort_segment_kernel below).  Longer segments, or more
// buckets, take a least-significant-digit radix sort: one stable counting pass
// per 8-bit digit of the bucket id (one pass up to 256 buckets, two up to
// 65536), each pass in three steps over tiles of kRadixTile elements:
//   1. count:   per (segment, tile) histogram of the digit, stored digit-major:
//               cnt[seg][digit][tile];
//   2. scan:    exclusive prefix sum over each segment's cnt array, which makes
//               cnt[seg][d][t] the first slot of digit d's elements of tile t;
//               the array is cut into chunks, summed by one launch and scanned
//               by the next from the sum of the chunks before each, so that a
//               segment's scan spreads over several SMs;
//   3. scatter: a 32-warp CTA per tile: each warp counts its range of the tile,
//               the CTA turns the (digit, warp) counts into offsets inside the
//               tile (digit-major, so warp ranges stay in order), and each warp
//               places its range in order, ranking equal digits inside a group
//               of 32 with a warp match.
// The first pass reads the bucket ids and writes (bucket, position) pairs in
// digit order to the workspace; the last pass writes perm (and inv).  Ids
// outside [0, n_buckets) are skipped by the first pass and recorded in the
// device status word; the scan of the first pass keeps each segment's count of
// valid ids, so the later pass reads only those.  No step waits on another CTA,
// so there is no inter-CTA spin.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kRadixBits = 8;
constexpr int kRadixDigits = 1 << kRadixBits;
constexpr int kRadixWarps = 32;
constexpr int kRadixPerWarp = 128;                          // 4 groups of 32 per warp
constexpr int kRadixTile = kRadixWarps * kRadixPerWarp;     // 4096 elements per CTA
constexpr int kScanMaxChunks = 64;                          // scan chunks per segment
constexpr int kScanMinChunk = 16384;                        // counters per scan chunk, at least

__host__ inline int radix_passes(int n_buckets) { return n_buckets <= kRadixDigits ? 1 : 2; }
__host__ inline int radix_tiles(int L) { return (L + kRadixTile - 1) / kRadixTile; }

// Scan chunks per segment for n counters per segment: enough CTAs for about two per SM, none
// shorter than kScanMinChunk counters.
__host__ inline int sort_scan_chunks(long long segs, long long n) {
  long long c = (296 + segs - 1) / segs;
  c = c < (long long)kScanMaxChunks ? c : (long long)kScanMaxChunks;
  const long long by_size = (n + kScanMinChunk - 1) / kScanMinChunk;
  c = c < by_size ? c : by_size;
  return (int)(c > 0 ? c : 1);
}

// Workspace of the radix sort, in 32-bit words: counters [seg][digit][tile], scan chunk sums
// [seg][chunk], valid ids per segment [seg], and, with two passes, the first pass's bucket ids and
// positions [seg][L] each.
struct RadixWs {
  long long cnt, sums, valid, keys, pos, words;
};
__host__ inline RadixWs radix_ws(long long segs, int L, int n_buckets) {
  RadixWs w;
  const long long n = (long long)kRadixDigits * radix_tiles(L);
  w.cnt = 0;
  w.sums = w.cnt + segs * n;
  w.valid = w.sums + segs * sort_scan_chunks(segs, n);
  w.keys = w.valid + segs;
  w.keys = (w.keys + 3) & ~3ll;  // 16-byte aligned
  const long long pair = radix_passes(n_buckets) > 1 ? segs * (long long)L : 0;
  w.pos = w.keys + pair;
  w.words = w.pos + pair;
  return w;
}

// 1. digit histogram of one tile (FIRST: the keys are the bucket ids, each checked; later passes
// read the first pass's ids, only the segment's valid ones).
template <bool FIRST>
__global__ void __launch_bounds__(1024)
radix_count_kernel(const int32_t* __restrict__ keys, int L, int n_buckets, int shift,
                   const uint32_t* __restrict__ n_valid, uint32_t* __restrict__ cnt) {
  __shared__ uint32_t hist[kRadixDigits];
  const long long seg = blockIdx.x;
  const int tile = blockIdx.y, nt = gridDim.y;
  const int n = FIRST ? L : (int)n_valid[seg];
  if (threadIdx.x < kRadixDigits) hist[threadIdx.x] = 0;
  __syncthreads();
  const int32_t* src = keys + seg * (long long)L;
  const int lo = tile * kRadixTile, hi = min(n, lo + kRadixTile);
  for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    const int k = src[i];
    if (FIRST && (unsigned)k >= (unsigned)n_buckets) {
      record_error(LSH_ERR_INVALID_ARG);
      continue;
    }
    atomicAdd(&hist[(k >> shift) & (kRadixDigits - 1)], 1u);
  }
  __syncthreads();
  if (threadIdx.x < kRadixDigits)
    cnt[(seg * kRadixDigits + threadIdx.x) * nt + tile] = hist[threadIdx.x];
}

// 2a. sum of scan chunk blockIdx.y of segment blockIdx.x: counters [c C, min(n, (c + 1) C)).
__global__ void __launch_bounds__(1024)
sort_chunk_sum_kernel(const uint32_t* __restrict__ cnt, long long n, long long C, uint32_t* __restrict__ sums) {
  __shared__ uint32_t warp_sums[32];
  const long long seg = blockIdx.x;
  const int c = blockIdx.y;
  const uint32_t* a = cnt + (size_t)seg * n;
  const long long lo = (long long)c * C, hi = lo + C < n ? lo + C : n;
  uint32_t v = 0;
  for (long long i = lo + threadIdx.x; i < hi; i += 1024) v += a[i];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_sums[lane];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) w += __shfl_xor_sync(0xffffffffu, w, off);
    if (lane == 0) sums[seg * gridDim.y + c] = w;
  }
}

// 2b. exclusive scan of scan chunk blockIdx.y of segment blockIdx.x (1024 threads, 4 counters per
// thread per step, carried across steps), starting from the sum of the segment's earlier chunks; the
// last chunk stores the segment's total (nullable).
__global__ void __launch_bounds__(1024)
sort_scan_kernel(uint32_t* __restrict__ cnt, long long n, long long C, const uint32_t* __restrict__ sums,
                 uint32_t* __restrict__ total) {
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t carry_s;
  const long long seg = blockIdx.x;
  const int c = blockIdx.y;
  uint32_t* a = cnt + (size_t)seg * n;
  const long long lo = (long long)c * C, hi = lo + C < n ? lo + C : n;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp == 0) {
    uint32_t base = 0;
    for (int k = lane; k < c; k += 32) base += sums[seg * gridDim.y + k];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) base += __shfl_xor_sync(0xffffffffu, base, off);
    if (lane == 0) carry_s = base;
  }
  __syncthreads();
  for (long long base = lo; base < hi; base += 4 * 1024) {
    const long long i0 = base + 4ll * threadIdx.x;
    uint32_t x[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) x[q] = (i0 + q < hi) ? a[i0 + q] : 0u;
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
      if (i0 + q < hi) a[i0 + q] = run;
      run += x[q];
    }
    __syncthreads();
    if (threadIdx.x == 1023) carry_s = run;
    __syncthreads();
  }
  if (total && c == (int)gridDim.y - 1 && threadIdx.x == 0) total[seg] = carry_s;  // the segment's sum
}

// 3. stable scatter of one tile by a CTA of kRadixWarps warps (FIRST: keys are the bucket ids and
// positions their indices; LAST: the output is perm and inv, else the (id, position) pairs for the
// next pass).
template <bool FIRST, bool LAST>
__global__ void __launch_bounds__(kRadixWarps * 32)
radix_scatter_kernel(const int32_t* __restrict__ keys, const int32_t* __restrict__ pos_in, int L, int n_buckets,
                     int shift, const uint32_t* __restrict__ n_valid, const uint32_t* __restrict__ cnt,
                     int32_t* __restrict__ key_out, int32_t* __restrict__ pos_out, int32_t* __restrict__ inv) {
  __shared__ uint32_t wh[kRadixWarps * kRadixDigits / 2];  // uint16 [warp][digit]: counts, then offsets
  __shared__ uint32_t base[kRadixDigits];                  // the tile's first slot of each digit
  uint16_t* whist = reinterpret_cast<uint16_t*>(wh);
  const long long seg = blockIdx.x;
  const int tile = blockIdx.y, nt = gridDim.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = FIRST ? L : (int)n_valid[seg];
  const int lo = tile * kRadixTile + warp * kRadixPerWarp;
  const int hi = min(n, lo + kRadixPerWarp);
  for (int i = threadIdx.x; i < kRadixWarps * kRadixDigits / 2; i += blockDim.x) wh[i] = 0;
  if (threadIdx.x < kRadixDigits) base[threadIdx.x] = cnt[(seg * kRadixDigits + threadIdx.x) * nt + tile];
  __syncthreads();
  // the warp's ids (four groups of 32, loaded together), their digits and validity
  const int32_t* src = keys + seg * (long long)L;
  int key[4], dig[4];
  bool ok[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = lo + 32 * k + lane;
    key[k] = i < hi ? src[i] : -1;
    ok[k] = i < hi && (!FIRST || (unsigned)key[k] < (unsigned)n_buckets);
    dig[k] = (key[k] >> shift) & (kRadixDigits - 1);
  }
  // a. per-warp digit counts (two digits per 32-bit word; a warp counts at most 128, no carry)
  uint32_t* my_words = wh + warp * kRadixDigits / 2;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (ok[k]) atomicAdd(&my_words[dig[k] >> 1], 1u << (16 * (dig[k] & 1)));
  __syncthreads();
  // b. per digit, exclusive offsets over the warps (in warp = position order), below kRadixTile
  if (threadIdx.x < kRadixDigits) {
    uint32_t run = 0;
    for (int w = 0; w < kRadixWarps; ++w) {
      const uint32_t c = whist[w * kRadixDigits + threadIdx.x];
      whist[w * kRadixDigits + threadIdx.x] = (uint16_t)run;
      run += c;
    }
  }
  __syncthreads();
  // c. stable placement of the warp's range
  uint16_t* my = whist + warp * kRadixDigits;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int32_t* psrc = FIRST ? nullptr : pos_in + seg * (long long)L;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = lo + 32 * k + lane;
    const unsigned vmask = __ballot_sync(0xffffffffu, ok[k]);
    unsigned peers = 0;
    uint32_t slot = 0;
    if (ok[k]) {
      peers = __match_any_sync(vmask, dig[k]);
      slot = base[dig[k]] + my[dig[k]] + __popc(peers & lt_mask);
    }
    __syncwarp();
    if (ok[k] && (peers & lt_mask) == 0) my[dig[k]] = (uint16_t)(my[dig[k]] + __popc(peers));
    __syncwarp();
    if (ok[k]) {
      const int pos = FIRST ? i : psrc[i];
      if (LAST) {
        pos_out[seg * (long long)L + slot] = pos;
        if (inv) inv[seg * (long long)L + pos] = (int32_t)slot;
      } else {
        key_out[seg * (long long)L + slot] = key[k];
        pos_out[seg * (long long)L + slot] = pos;
      }
    }
  }
}

// Whole-segment sort in one CTA (L <= 65536, n_buckets <= 1024): each of the
// 32 warps counts a contiguous range of the segment into its own histogram, the
// CTA turns the (bucket, warp) counts into exclusive offsets (bucket-major, so
// warp ranges stay in position order inside a bucket), and each warp then
// places its range in order with the warp-match ranking of
// radix_scatter_kernel.  Counts, offsets and sorted slots are all below 65536,
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

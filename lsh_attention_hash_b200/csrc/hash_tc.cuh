// Angular LSH hash on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Ultralytics glossary "Reformer", section "Atencao LSH": bucket = position of
// the largest value of [xR, -xR] for a random projection R per round.
//
// Served case: bf16 rows, D in {64, 128}, n_buckets/2 = `half` 32, or a
// multiple of 64 with half <= 256 or half % 256 == 0 (half = 32: R[round] is
// copied into a 64-column tile whose upper 32 columns are zero, by plain loads).  Each persistent CTA owns one round
// and 128-row tiles of QK stream through a two-stage TMA ring.  R[round] (MN-
// major, 128-byte swizzle) either stays in shared memory, loaded once by TMA
// (D * half * 2 <= 128 KB), or, for larger bucket counts (RS > 0), streams
// through an RS-stage TMA ring in chunks of NC columns for every tile (it is
// re-read from L2, where the rounds' projections stay).  p = x R accumulates in
// fp32 in TMEM (two buffers of NC <= 256 columns, so the next chunk's UMMA
// overlaps the current epilogue).
//
// Epilogue (one row per thread): the bucket is argmax over [p, -p], i.e. the
// largest |p_k| and its sign.  Values are handled in groups of 16: the key of
// p_k is |p_k| with its 4 lowest mantissa bits replaced by (15 - k % 16), so a
// 3-input max tree over the keys yields the group's largest |p| (to 2^-19
// relative, far below the 1e-5 near-tie threshold) together with its
// position (ties prefer the lower column); a max tree over the raw values of
// the winning group tells its sign.  The exact top-two |p| for the near-tie
// flag are tracked only when that output is requested.
//
// Warps: 0 TMA producer, 1 UMMA issuer, then 4 * SPLIT epilogue warps.  SPLIT
// epilogue warps share each TMEM lane quarter (32 rows) and take 1/SPLIT of
// the columns of every accumulator chunk each; at the end of a tile the other
// parts' row states go through shared memory to part 0, which merges and
// stores.
#pragma once

#include "tc_common.cuh"

namespace lsh {
namespace hash_tc {

constexpr int kRows = 128;
__host__ __device__ constexpr int threads_for(int split) { return 64 + 128 * split; }
constexpr int kStages = 2;

constexpr int kMaxRS = 4;  // stages of the streamed projection ring

template <int D>
struct Layout {
  static constexpr uint32_t kHalfBytes = kRows * 128;           // 128 rows x 64 bf16
  static constexpr uint32_t kStageBytes = (D / 64) * kHalfBytes;
  static constexpr uint32_t kA = 0;
  static constexpr uint32_t kR = kStages * kStageBytes;          // R: (columns / 64) boxes of D x 128 B
  // resident: all of R[round] (at least one 64-column box); streamed: RS chunks of nc columns
  __host__ __device__ static constexpr uint32_t r_bytes(int half, int nc, int rs) {
    return rs ? (uint32_t)rs * D * nc * 2 : (uint32_t)D * (half < 64 ? 64 : half) * 2;
  }
  __host__ __device__ static constexpr uint32_t bar_off(int half, int nc, int rs) { return kR + r_bytes(half, nc, rs); }
  // a_full[2] a_empty[2] acc_full[2] acc_empty[2] r_full done part_done[2] merged[2]
  // then the streamed ring's rs_full[kMaxRS] rs_empty[kMaxRS]
  static constexpr int kNumBars = 14 + 2 * kMaxRS;
  // row states of parts 1..3: [2 tile parities][3 parts][5 fields][128 rows] x 4 B
  __host__ __device__ static constexpr uint32_t xchg_off(int half, int nc, int rs) {
    return bar_off(half, nc, rs) + kNumBars * 8 + 16;
  }
  __host__ __device__ static constexpr uint32_t smem_bytes(int half, int nc, int rs) {
    return xchg_off(half, nc, rs) + 2 * 3 * 5 * kRows * 4 + 1024;
  }
};

struct Params {
  const __nv_bfloat16* r;  // [n_rounds][D][half] (the 32-column case copies it by plain loads)
  int32_t* buckets;    // [B*H][n_rounds][L]
  uint8_t* near_tie;   // same, nullable
  long long nrows;     // B*H*L
  int L;
  int n_rounds;
  int half;
  int nchunks;         // half / NC
  int per_round;       // CTAs per round
  long long n_tiles;
  uint32_t key_mask;   // 0x7FFFFFF0: |p| without its 4 lowest mantissa bits
};

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max over 16 values with 3-input maxima
__device__ __forceinline__ float max16(const float* v) {
  const float a = max3(v[0], v[1], v[2]), b = max3(v[3], v[4], v[5]), c = max3(v[6], v[7], v[8]);
  const float d = max3(v[9], v[10], v[11]), e = max3(v[12], v[13], v[14]);
  return max3(max3(a, b, c), d, fmaxf(e, v[15]));
}

struct RowState {
  float best_key;   // largest key so far
  int best_g;       // its group (16 columns) within the round
  float best_raw;   // largest raw value of that group
  float v1, v2;     // exact top-two |p| (near-tie flag only)
  float best_abs;   // largest exact |p| so far (wide rounds)
};

// `mask` is 0x7FFFFFF0, passed in at run time: with the mask in a register
// (or constant operand) and 15 - j as the immediate, each key is a single
// three-input logic operation instead of two.
template <bool FLAG>
__device__ __forceinline__ void process16(RowState& st, const uint32_t* raw, int g, uint32_t mask) {
  float key[16], val[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    val[j] = __uint_as_float(raw[j]);
    key[j] = __uint_as_float((raw[j] & mask) | (uint32_t)(15 - j));
  }
  const float gk = max16(key);
  const float gr = max16(val);
  const bool gt = gk > st.best_key;
  st.best_key = gt ? gk : st.best_key;
  st.best_g = gt ? g : st.best_g;
  st.best_raw = gt ? gr : st.best_raw;
  if (FLAG) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float a = fabsf(val[j]);
      st.v2 = fmaxf(st.v2, fminf(st.v1, a));
      st.v1 = fmaxf(st.v1, a);
    }
  }
}

// Wide rounds (thousands of columns per row): after the first few dozen groups a group rarely holds
// a new row maximum, so each group first takes only its exact largest |p| (a 3-input max tree
// over the absolute values) and the keyed pass above runs, for the whole warp, only when some lane
// of the warp has a new maximum.  The row's best group is then the one with the largest exact
// |p|, and within it the keyed pass picks the column, so the result can differ from the keyed pass
// over every group only where two values agree to 2^-19 relative, inside the near-tie band.
__device__ __forceinline__ void process16_wide(RowState& st, const uint32_t* raw, int g, uint32_t mask) {
  float a[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) a[j] = fabsf(__uint_as_float(raw[j]));
  const float gm = max16(a);
  const bool rec = gm > st.best_abs;
  if (__any_sync(0xffffffffu, rec)) {
    float key[16], val[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      val[j] = __uint_as_float(raw[j]);
      key[j] = __uint_as_float((raw[j] & mask) | (uint32_t)(15 - j));
    }
    const float gk = max16(key);
    const float gr = max16(val);
    if (rec) {
      st.best_key = gk;
      st.best_g = g;
      st.best_raw = gr;
      st.best_abs = gm;
    }
  }
}

template <int D, int NC, bool FLAG, int SPLIT, int RS, bool WIDE = false>
__global__ void __launch_bounds__(threads_for(SPLIT), 1)
hash_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_r,
               const Params p) {
  using Lay = Layout<D>;
  constexpr uint32_t kRS = RS > 0 ? RS : 1;  // ring stages as a divisor (the resident layout has none)
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte-aligned base as an offset from the shared array itself (not an integer
  // cast), so that every access through it stays a shared-memory access
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bar_off(p.half, NC, RS));
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + 2;
  uint64_t* acc_full = bars + 4;
  uint64_t* acc_empty = bars + 6;
  uint64_t* r_full = bars + 8;
  uint64_t* done_bar = bars + 9;
  uint64_t* part_done = bars + 10;  // [2] parts 1.. states written ((SPLIT-1) * 128 arrivals)
  uint64_t* merged = bars + 12;     // [2] those states consumed (128 arrivals)
  uint64_t* rs_full = bars + 14;    // [RS] streamed R chunk landed
  uint64_t* rs_empty = rs_full + kMaxRS;  // [RS] its UMMAs retired
  float* xchg = reinterpret_cast<float*>(smem + Lay::xchg_off(p.half, NC, RS));
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + Lay::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + Lay::kNumBars) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int round = blockIdx.x % p.n_rounds;
  const int first_tile = blockIdx.x / p.n_rounds;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&a_full[i], 1);
      tc::mbar_init(&a_empty[i], 1);
      tc::mbar_init(&acc_full[i], 1);
      tc::mbar_init(&acc_empty[i], 128 * SPLIT);
      tc::mbar_init(&part_done[i], SPLIT > 1 ? 128 * (SPLIT - 1) : 1);  // unused with one part
      tc::mbar_init(&merged[i], 128);
    }
    tc::mbar_init(r_full, 1);
    tc::mbar_init(done_bar, 1);
    for (int i = 0; i < RS; ++i) {
      tc::mbar_init(&rs_full[i], 1);
      tc::mbar_init(&rs_empty[i], 1);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_holder, 2 * NC < 32 ? 32 : 2 * NC);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (RS == 0 && p.half < 64) {
      // R[round] (D x 32) into one 64-column MN-major tile with the 128-byte
      // swizzle: row k holds columns 0..31 in its 16-byte pieces 0..3, pieces
      // 4..7 are zero (the UMMA reads only N = 32 columns of it)
      const __nv_bfloat16* rsrc = p.r + (size_t)round * D * p.half;
      for (int idx = lane; idx < D * 8; idx += 32) {
        const int k = idx >> 3, c = idx & 7;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (c < 4) val = *reinterpret_cast<const uint4*>(rsrc + (size_t)k * p.half + c * 8);
        *reinterpret_cast<uint4*>(smem + Lay::kR + k * 128 + ((c ^ (k & 7)) << 4)) = val;
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(r_full);
    }
    if (lane == 0) {
      tc::prefetch_tensormap(&map_x);
      tc::prefetch_tensormap(&map_r);
      if (RS == 0 && p.half >= 64) {  // R[round] resident: loaded once
        tc::mbar_arrive_expect_tx(r_full, (uint32_t)D * p.half * 2);
        for (int b = 0; b < p.half / 64; ++b)
          tc::tma_load_2d(smem + Lay::kR + b * D * 128, &map_r, r_full, b * 64, round * D);
      }
      uint32_t it = 0, rq = 0;
      bool ok = true;
      for (long long tile = first_tile; tile < p.n_tiles; tile += p.per_round, ++it) {
        const int s = it % kStages;
        ok = tc::mbar_wait(&a_empty[s], ((it / kStages) & 1) ^ 1, abort_flag);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(&a_full[s], kRows * D * 2);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tc::tma_load_2d(smem + Lay::kA + s * Lay::kStageBytes + h * Lay::kHalfBytes, &map_x, &a_full[s], h * 64,
                          (int)(tile * kRows));
        if (RS > 0) {  // the tile's pass over R[round], chunk by chunk
          for (int c = 0; ok && c < p.nchunks; ++c, ++rq) {
            const int sr = rq % kRS;
            ok = tc::mbar_wait(&rs_empty[sr], ((rq / kRS) & 1) ^ 1, abort_flag);
            if (!ok) break;
            tc::mbar_arrive_expect_tx(&rs_full[sr], (uint32_t)D * NC * 2);
#pragma unroll
            for (int b = 0; b < NC / 64; ++b)
              tc::tma_load_2d(smem + Lay::kR + sr * (D * NC * 2) + b * D * 128, &map_r, &rs_full[sr],
                              c * NC + b * 64, round * D);
          }
          if (!ok) break;
        }
      }
      // never leave with copies in flight
      for (uint32_t k = (it > kStages ? it - kStages : 0); k < it; ++k) {
        const unsigned long long t0 = tc::globaltimer();
        while (!tc::mbar_try_wait(&a_full[k % kStages], (k / kStages) & 1))
          if (tc::globaltimer() - t0 > tc::kWaitNs / 16) break;
      }
      if (RS == 0 && p.half >= 64) {
        const unsigned long long t0 = tc::globaltimer();
        while (!tc::mbar_try_wait(r_full, 0))
          if (tc::globaltimer() - t0 > tc::kWaitNs / 16) break;
      }
      for (uint32_t k = (rq > (uint32_t)RS ? rq - RS : 0); k < rq; ++k) {
        const unsigned long long t0 = tc::globaltimer();
        while (!tc::mbar_try_wait(&rs_full[k % kRS], (k / kRS) & 1))
          if (tc::globaltimer() - t0 > tc::kWaitNs / 16) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, NC, 0, 1);
      const uint32_t a0 = tc::smem_u32(smem + Lay::kA);
      const uint32_t r0 = tc::smem_u32(smem + Lay::kR);
      bool ok = RS > 0 || tc::mbar_wait(r_full, 0, abort_flag);
      uint32_t it = 0, seq = 0, rq = 0;
      for (long long tile = first_tile; ok && tile < p.n_tiles; tile += p.per_round, ++it) {
        const int s = it % kStages;
        ok = tc::mbar_wait(&a_full[s], (it / kStages) & 1, abort_flag);
        if (!ok) break;
        for (int c = 0; c < p.nchunks; ++c, ++seq) {
          const int b = seq & 1;
          const int sr = RS > 0 ? (int)(rq % kRS) : 0;
          if (RS > 0) {
            ok = tc::mbar_wait(&rs_full[sr], (rq / kRS) & 1, abort_flag);
            if (!ok) break;
          }
          ok = tc::mbar_wait(&acc_empty[b], ((seq >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
          tc::tc_fence_after();
          // chunk c of R[round]: resident at its offset, or the ring stage it streamed into
          const uint32_t rbase = RS > 0 ? r0 + sr * (D * NC * 2) : r0 + (c * (NC / 64)) * D * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(a0 + s * Lay::kStageBytes + (kk >> 2) * Lay::kHalfBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(rbase + kk * 2048, D * 128, 1024);
            tc::umma_ss(tmem + b * NC, ad, bd, idesc, kk > 0);
          }
          tc::umma_commit(&acc_full[b]);
          if (RS > 0) {
            tc::umma_commit(&rs_empty[sr]);
            ++rq;
          }
        }
        if (!ok) break;
        tc::umma_commit(&a_empty[s]);
      }
      tc::umma_commit(done_bar);
      const unsigned long long t0 = tc::globaltimer();
      while (!tc::mbar_try_wait(done_bar, 0))
        if (tc::globaltimer() - t0 > tc::kWaitNs / 16) break;
    }
    __syncwarp();
  } else {
    constexpr int kCols = NC / SPLIT;    // columns of every chunk handled by one part
    const int q = warp & 3;
    const int ch = (warp - 2) >> 2;      // part of every chunk
    const int r = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t seq = 0, it = 0;
    bool ok = true;
    for (long long tile = first_tile; ok && tile < p.n_tiles; tile += p.per_round, ++it) {
      RowState st{-1.f, 0, 0.f, -INFINITY, -INFINITY, -1.f};
      for (int c = 0; c < p.nchunks; ++c, ++seq) {
        const int b = seq & 1;
        ok = att_tc::warp_wait(&acc_full[b], (seq >> 1) & 1, abort_flag);
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int piece = 0; piece < kCols / 32; ++piece) {
          uint32_t raw[32];
          const int col = ch * kCols + piece * 32;
          tc::tmem_ld32(lane_base + tmem + b * NC + col, raw);
          tc::tmem_wait_ld();
          const int g = (c * NC + col) >> 4;
          if (WIDE) {
            process16_wide(st, raw, g, p.key_mask);
            process16_wide(st, raw + 16, g + 1, p.key_mask);
          } else {
            process16<FLAG>(st, raw, g, p.key_mask);
            process16<FLAG>(st, raw + 16, g + 1, p.key_mask);
          }
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&acc_empty[b]);
      }
      if (!ok) break;
      const int tp = it & 1;
      if (SPLIT > 1 && ch > 0) {
        float* xs = xchg + (tp * 3 + (ch - 1)) * 5 * kRows;
        ok = att_tc::warp_wait(&merged[tp], ((it >> 1) & 1) ^ 1, abort_flag);
        if (!ok) break;
        xs[r] = st.best_key;
        xs[kRows + r] = __int_as_float(st.best_g);
        xs[2 * kRows + r] = st.best_raw;
        xs[3 * kRows + r] = st.v1;
        xs[4 * kRows + r] = st.v2;
        tc::mbar_arrive(&part_done[tp]);
        continue;
      }
      if (SPLIT > 1) {
        ok = att_tc::warp_wait(&part_done[tp], (it >> 1) & 1, abort_flag);
        if (!ok) break;
      }
#pragma unroll
      for (int o = 0; o < SPLIT - 1; ++o) {
        const float* xs = xchg + (tp * 3 + o) * 5 * kRows;
        const float o_key = xs[r];
        const int o_g = __float_as_int(xs[kRows + r]);
        // the parts cover disjoint groups; on equal keys the lower group wins
        if (o_key > st.best_key || (o_key == st.best_key && o_g < st.best_g)) {
          st.best_key = o_key;
          st.best_g = o_g;
          st.best_raw = xs[2 * kRows + r];
        }
        if (FLAG) {
          const float o_v1 = xs[3 * kRows + r], o_v2 = xs[4 * kRows + r];
          st.v2 = fmaxf(fmaxf(st.v2, o_v2), fminf(st.v1, o_v1));
          st.v1 = fmaxf(st.v1, o_v1);
        }
      }
      if (SPLIT > 1) tc::mbar_arrive(&merged[tp]);
      const long long row = tile * kRows + r;
      if (row < p.nrows) {
        const uint32_t kb = __float_as_uint(st.best_key);
        const int k = st.best_g * 16 + (15 - (int)(kb & 15u));
        const bool pos = st.best_raw >= 0.f && ((__float_as_uint(st.best_raw) & 0x7FFFFFF0u) == (kb & 0x7FFFFFF0u));
        const long long bh = row / p.L, l = row - bh * p.L;
        const size_t o = ((size_t)bh * p.n_rounds + round) * p.L + l;
        p.buckets[o] = pos ? k : k + p.half;
        if (FLAG) {
          const float u1 = st.v1, u2 = fmaxf(st.v2, -st.v1);
          p.near_tie[o] = (u1 - u2) < kTieRel * fmaxf(u1, 1e-30f) ? 1 : 0;
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 2 * NC < 32 ? 32 : 2 * NC);
  }
}

}  // namespace hash_tc
}  // namespace lsh

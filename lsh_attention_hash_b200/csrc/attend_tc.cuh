// Chunk attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// twgreatdaily ICLR 2020 Reformer article, section "1 LSH Attention": after
// the (bucket, position) sort the sequence is cut into chunks; a chunk's
// queries attend to their own chunk and the previous one (no wrap-around for
// chunk 0); the output is the sum over the admissible keys of exp(logit) v
// divided by the partition function; Q = K, keys length-normalised; a token
// does not attend to itself while it has another key.  Scale 1/sqrt(d_k):
// ai-scholar.tech Reformer article, "Transformerの問題点とは".
//
// Served case: bf16 rows, chunk 64, D in {64, 128}.  One step takes two
// consecutive sorted chunks (2j, 2j+1) as 128 query rows and the window
// chunks (2j-1, 2j, 2j+1) as 192 keys:
//   S[128 x 192] = Q K^T        two UMMAs (N = 64 for chunk 2j-1, N = 128 for
//                                the pair itself, whose rows are also Q)
//   row r sees keys [64*(r>=64), 64*(r>=64) + 128); its own key is 64 + r%64
//   P = exp2(S * s_j - max) in bf16, written back over S in TMEM
//   O[128 x D] = P V            UMMA with A = P from TMEM, B = V (MN-major)
// and the rows go back to their original positions perm[s].
//
// Warp roles (192 threads, persistent CTAs, one per SM):
//   warp 0     producer: reads perm, gathers the QK and V rows of each chunk
//              with TMA tile::gather4 (128-byte swizzled, K-major) into a ring
//              of three 128-row slots;
//   warp 1     TMEM owner and single-thread UMMA issuer;
//   warps 2-5  one query row per thread: key lengths, softmax, P, epilogue.
// TMEM: two S/P buffers of 192 columns and one O buffer (512 columns).
// Every wait is bounded (tc::mbar_wait); a timeout unwinds the CTA cleanly.
#pragma once

#include "tc_common.cuh"

namespace lsh {
namespace att_tc {

constexpr int kC = 64;         // chunk length served
constexpr int kRows = 128;     // query rows per step
constexpr int kSlots = 3;      // 128-row slots in the shared-memory ring
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCols = 192;  // one S/P buffer
constexpr uint32_t kOCol = 2 * kSCols;

template <int D>
struct Layout {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kHalfBytes = kRows * 128;          // 128 rows x 64 bf16
  static constexpr uint32_t kSlotBytes = kHalves * kHalfBytes; // one tensor, one slot
  static constexpr uint32_t kQK = 0;
  static constexpr uint32_t kV = kSlots * kSlotBytes;
  static constexpr uint32_t kPerm = 2 * kSlots * kSlotBytes;        // int32 [kSlots][128]
  static constexpr uint32_t kColMul = kPerm + kSlots * kRows * 4;   // float [kSlots][128]
  static constexpr uint32_t kBar = kColMul + kSlots * kRows * 4;
  // full[3] empty[3] s_full[2] p_ready[2] o_full o_empty cm_ready done
  static constexpr int kNumBars = 14;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;   // tmem base, abort flag
  static constexpr uint32_t kBytes = kMisc + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;         // slack for 1024-byte alignment
};

struct Params {
  const int32_t* perm;   // [segs][L]
  void* out;             // [segs][L][D]
  float* lse;            // [segs][L]
  int L;
  int n_rounds;
  int n_chunks;          // L / 64
  int n_steps;           // ceil(n_chunks / 2)
  int run;               // steps per work unit
  int units_per_seg;
  long long n_units;
  int self_mask;
  float colscale;        // logit scale * log2(e)
  int sorted_input;      // rows of the tensor maps are [seg][slot] instead of [bh][pos]
};

// Warp-uniform bounded wait: every lane acquires the phase itself, lane 0
// decides on abort / timeout so that the warp leaves together.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  bool done = tc::mbar_try_wait(bar, parity);
  if (__all_sync(0xffffffffu, done)) return true;
  const unsigned long long t0 = tc::globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (!done) done = tc::mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    if ((i & 31u) == 0) {
      int bail = 0;
      if ((threadIdx.x & 31) == 0) {
        if (*abort_flag) {
          bail = 1;
        } else if (tc::globaltimer() - t0 > tc::kWaitNs) {
          *abort_flag = 1;
          record_error(LSH_ERR_TIMEOUT);
          bail = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, bail, 0)) return false;
    }
  }
}

// Bounded wait that ignores the abort flag (used to drain in-flight copies and MMAs).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = tc::globaltimer();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (tc::globaltimer() - t0 > tc::kWaitNs / 16) {
      record_error(LSH_ERR_TIMEOUT);
      return;
    }
  }
}

struct Unit {
  long long seg;
  int j0, j1;
};

__device__ __forceinline__ Unit decode_unit(const Params& p, long long u) {
  Unit w;
  w.seg = u / p.units_per_seg;
  const int run_i = (int)(u - w.seg * p.units_per_seg);
  w.j0 = run_i * p.run;
  w.j1 = min(w.j0 + p.run, p.n_steps);
  return w;
}

// Loads `nrows` rows (64 or 128) of chunks (cA for local rows [row0, row0+64),
// cB for [row0+64, row0+128)) into slot `slot`, rows starting at `row0`.
template <int D>
__device__ __forceinline__ void producer_fill(const Params& p, const CUtensorMap* mqk, const CUtensorMap* mv,
                                              uint8_t* smem, uint64_t* full_bar, int slot, long long seg,
                                              int row0, int nrows, int cA, int cB) {
  using Lay = Layout<D>;
  const int lane = threadIdx.x & 31;
  int32_t* perm_s = reinterpret_cast<int32_t*>(smem + Lay::kPerm) + slot * kRows;
  const long long bh = seg / p.n_rounds;
  const int32_t* pseg = p.perm + seg * p.L;
  int grow[4];
  const bool active = lane * 4 < nrows;
  if (active) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int rr = row0 + lane * 4 + k;                 // local row in the slot
      const int chunk = (rr - row0) < 64 ? cA : cB;
      const int s = chunk * kC + (rr & 63);
      const int pos = pseg[s];
      perm_s[rr] = pos;
      grow[k] = p.sorted_input ? (int)(seg * p.L + s) : (int)(bh * p.L + pos);
    }
  }
  __syncwarp();
  if (lane == 0) tc::mbar_arrive_expect_tx(full_bar, (uint32_t)(nrows * D * 2 * 2));
  __syncwarp();
  if (active) {
    const int rr = row0 + lane * 4;
#pragma unroll
    for (int h = 0; h < Lay::kHalves; ++h) {
      uint8_t* dq = smem + Lay::kQK + slot * Lay::kSlotBytes + h * Lay::kHalfBytes + rr * 128;
      uint8_t* dv = smem + Lay::kV + slot * Lay::kSlotBytes + h * Lay::kHalfBytes + rr * 128;
      tc::tma_gather4(dq, mqk, full_bar, h * 64, grow[0], grow[1], grow[2], grow[3]);
      tc::tma_gather4(dv, mv, full_bar, h * 64, grow[0], grow[1], grow[2], grow[3]);
    }
  }
}

// scale * log2(e) / ||row||, read from the swizzled row of a QK slot (the
// 16-byte pieces of a row stay inside its 128-byte line, in permuted order).
template <int D>
__device__ __forceinline__ float row_colmul(const uint8_t* qk_slot, int r, float colscale) {
  using Lay = Layout<D>;
  float ss = 0.f;
#pragma unroll
  for (int h = 0; h < Lay::kHalves; ++h) {
    const uint8_t* row = qk_slot + h * Lay::kHalfBytes + r * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float x[8];
      load8(reinterpret_cast<const __nv_bfloat16*>(row + ((c ^ (r & 7)) << 4)), x);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
    }
  }
  return colscale / fmaxf(sqrtf(ss), 1e-12f);
}

template <int D, typename TO>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap map_qk, const __grid_constant__ CUtensorMap map_v,
                 const Params p) {
  using Lay = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* full = bars;          // [3] slot filled (TMA bytes landed)
  uint64_t* empty = bars + 3;     // [3] slot released by the MMAs
  uint64_t* s_full = bars + 6;    // [2] S buffer computed
  uint64_t* p_ready = bars + 8;   // [2] P buffer written (128 arrivals)
  uint64_t* o_full = bars + 10;   // O computed
  uint64_t* o_empty = bars + 11;  // O read (128 arrivals)
  uint64_t* cm_ready = bars + 12; // key multipliers of the step written (128 arrivals)
  uint64_t* done_bar = bars + 13; // all MMAs retired
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);
  float* colmul = reinterpret_cast<float*>(smem + Lay::kColMul);
  const int32_t* perm_s = reinterpret_cast<const int32_t*>(smem + Lay::kPerm);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      tc::mbar_init(&full[i], 1);
      tc::mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&s_full[i], 1);
      tc::mbar_init(&p_ready[i], 128);
    }
    tc::mbar_init(o_full, 1);
    tc::mbar_init(o_empty, 128);
    tc::mbar_init(cm_ready, 128);
    tc::mbar_init(done_bar, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&map_qk);
    tc::prefetch_tensormap(&map_v);
  }
  if (warp == 1) tc::tmem_alloc(tmem_holder, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t f = 0;
    bool ok = true;
    for (long long u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const Unit w = decode_unit(p, u);
      {  // the chunk before the unit's first pair (chunk 0 again at the segment start: masked)
        const int slot = f % kSlots;
        ok = warp_wait(&empty[slot], ((f / kSlots) & 1) ^ 1, abort_flag);
        if (!ok) break;
        const int cp = w.j0 > 0 ? 2 * w.j0 - 1 : 0;
        producer_fill<D>(p, &map_qk, &map_v, smem, &full[slot], slot, w.seg, 64, 64, cp, cp);
        ++f;
      }
      for (int j = w.j0; j < w.j1; ++j) {
        const int slot = f % kSlots;
        ok = warp_wait(&empty[slot], ((f / kSlots) & 1) ^ 1, abort_flag);
        if (!ok) break;
        const int c0 = 2 * j;
        const int c1 = (2 * j + 1 < p.n_chunks) ? 2 * j + 1 : 2 * j;  // odd tail: repeat (rows unused)
        producer_fill<D>(p, &map_qk, &map_v, smem, &full[slot], slot, w.seg, 0, 128, c0, c1);
        ++f;
      }
    }
    // never leave with copies in flight
    if (lane == 0) {
      for (uint32_t k = (f > kSlots ? f - kSlots : 0); k < f; ++k) drain_wait(&full[k % kSlots], (k / kSlots) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      const uint32_t id_prev = tc::idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id_pair = tc::idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, D, 0, 1);
      const uint32_t qk0 = tc::smem_u32(smem + Lay::kQK);
      const uint32_t v0 = tc::smem_u32(smem + Lay::kV);
      uint32_t f = 0, t = 0;
      bool ok = true;
      for (long long u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        const Unit w = decode_unit(p, u);
        ++f;  // the unit's leading chunk fill
        for (int j = w.j0; j < w.j1; ++j) {
          const uint32_t fp = f - 1, fc = f;
          ++f;
          const int sp = fp % kSlots, sc = fc % kSlots;
          ok = tc::mbar_wait(&full[sp], (fp / kSlots) & 1, abort_flag) &&
               tc::mbar_wait(&full[sc], (fc / kSlots) & 1, abort_flag);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t sbuf = tmem + (t & 1) * kSCols;
          const uint32_t qk_c = qk0 + sc * Lay::kSlotBytes;
          const uint32_t qk_p = qk0 + sp * Lay::kSlotBytes + 64 * 128;  // rows 64..127 of the previous slot
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * Lay::kHalfBytes + (kk & 3) * 32;
            const uint64_t a = tc::sdesc_sw128(qk_c + koff, 16, 1024);
            const uint64_t bp = tc::sdesc_sw128(qk_p + koff, 16, 1024);
            tc::umma_ss(sbuf, a, bp, id_prev, kk > 0);
            tc::umma_ss(sbuf + 64, a, a, id_pair, kk > 0);
          }
          tc::umma_commit(&s_full[t & 1]);
          ok = tc::mbar_wait(&p_ready[t & 1], (t >> 1) & 1, abort_flag) &&
               tc::mbar_wait(o_empty, (t & 1) ^ 1, abort_flag);
          if (!ok) break;
          tc::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 12; ++kk) {
            const uint32_t vrow = kk < 4 ? v0 + sp * Lay::kSlotBytes + (64 + 16 * kk) * 128
                                         : v0 + sc * Lay::kSlotBytes + (16 * (kk - 4)) * 128;
            const uint64_t b = tc::sdesc_sw128(vrow, Lay::kHalfBytes, 1024);
            tc::umma_ts(tmem + kOCol, sbuf + kk * 8, b, id_pv, kk > 0);
          }
          tc::umma_commit(o_full);
          tc::umma_commit(&empty[sp]);
          ++t;
        }
        if (!ok) break;
        tc::umma_commit(&empty[(f - 1) % kSlots]);
      }
      tc::umma_commit(done_bar);
      drain_wait(done_bar, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;              // TMEM lane quarter of this warp
    const int r = q * 32 + lane;         // query row of the step
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const bool low = q < 2;              // rows 0..63: keys [0, 128); rows 64..127: keys [64, 192)
    const int self_i = 64 + (r & 63);    // own key, as an index into the row's 128 keys
    uint32_t f = 0, t = 0;
    bool ok = true;
    for (long long u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const Unit w = decode_unit(p, u);
      ++f;
      bool first = true;
      for (int j = w.j0; j < w.j1; ++j) {
        const uint32_t fp = f - 1, fc = f;
        ++f;
        const int sp = fp % kSlots, sc = fc % kSlots;
        ok = warp_wait(&full[sp], (fp / kSlots) & 1, abort_flag) &&
             warp_wait(&full[sc], (fc / kSlots) & 1, abort_flag);
        if (!ok) break;
        // key multipliers of the pair (and, at a unit start, of the leading chunk)
        colmul[sc * kRows + r] = row_colmul<D>(smem + Lay::kQK + sc * Lay::kSlotBytes, r, p.colscale);
        if (first && !low)
          colmul[sp * kRows + r] = row_colmul<D>(smem + Lay::kQK + sp * Lay::kSlotBytes, r, p.colscale);
        tc::mbar_arrive(cm_ready);
        const int chunk = 2 * j + (low ? 0 : 1);
        const bool valid = chunk < p.n_chunks;
        const int pos = perm_s[sc * kRows + r];
        ok = warp_wait(cm_ready, t & 1, abort_flag) && warp_wait(&s_full[t & 1], (t >> 1) & 1, abort_flag);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t sbuf = tmem + (t & 1) * kSCols;
        float x[128];
        {
          uint32_t raw[32];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            tc::tmem_ld32(lane_base + sbuf + (low ? 0 : 64) + 32 * g, raw);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) x[32 * g + e] = __uint_as_float(raw[e]);
          }
        }
        // multipliers: local key i -> low rows: i < 64 prev slot rows 64+i, else pair rows i-64;
        //                              high rows: pair rows i
        const float* cm_lo = low ? colmul + sp * kRows + 64 : colmul + sc * kRows;
        const float* cm_hi = low ? colmul + sc * kRows : colmul + sc * kRows + 64;
        const bool mask_prev = low && j == 0;  // chunk 0 has no previous chunk
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          float v = x[i] * (i < 64 ? cm_lo[i] : cm_hi[i - 64]);
          if ((p.self_mask && i == self_i) || (mask_prev && i < 64)) v = -INFINITY;
          x[i] = v;
          m = fmaxf(m, v);
        }
        float l = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float a = tc::ex2_approx(x[2 * i] - m);
          const float b = tc::ex2_approx(x[2 * i + 1] - m);
          l += a + b;
          pk[i] = tc::pack_bf16x2(a, b);
        }
        {
          uint32_t g0[32], g1[32], z[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            g0[e] = pk[e];
            g1[e] = pk[32 + e];
            z[e] = 0u;
          }
          if (low) {
            tc::tmem_st32(lane_base + sbuf + 0, g0);
            tc::tmem_st32(lane_base + sbuf + 32, g1);
            tc::tmem_st32(lane_base + sbuf + 64, z);
          } else {
            tc::tmem_st32(lane_base + sbuf + 0, z);
            tc::tmem_st32(lane_base + sbuf + 32, g0);
            tc::tmem_st32(lane_base + sbuf + 64, g1);
          }
          tc::tmem_wait_st();
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&p_ready[t & 1]);
        // epilogue: O row -> original position
        ok = warp_wait(o_full, t & 1, abort_flag);
        if (!ok) break;
        tc::tc_fence_after();
        float o[D];
        {
          uint32_t raw[32];
#pragma unroll
          for (int g = 0; g < D / 32; ++g) {
            tc::tmem_ld32(lane_base + tmem + kOCol + 32 * g, raw);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[32 * g + e] = __uint_as_float(raw[e]);
          }
        }
        tc::tc_fence_before();
        tc::mbar_arrive(o_empty);
        if (valid) {
          const float inv_l = 1.f / l;
          TO* dst = reinterpret_cast<TO*>(p.out) + (w.seg * p.L + pos) * (long long)D;
#pragma unroll
          for (int e = 0; e < D; e += 8) {
            float y[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) y[k] = o[e + k] * inv_l;
            store8(dst + e, y);
          }
          p.lse[w.seg * p.L + pos] = (m + __log2f(l)) * 0.6931471805599453f;
        }
        ++t;
        first = false;
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace att_tc
}  // namespace lsh

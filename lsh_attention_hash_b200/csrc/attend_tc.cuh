// Chunk attention on the 5th-generation tensor cores (tcgen05 + TMEM).
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
//   P = exp2(S * s_j - m) in bf16 (m a per-row shift), written back over the
//                                head of S in TMEM
//   O[128 x D] = P V            UMMA with A = P from TMEM, B = V (MN-major),
//                                accumulated behind P in the same TMEM buffer
// and the rows go back to their original positions perm[s].
//
// Warp roles (384 threads, persistent CTAs, one per SM, launched at 168
// registers per thread; warpgroup 0 gives registers to the softmax warpgroups
// with setmaxnreg, 104 / 192):
//   warps 0-1  producers: read perm and gather the QK and V rows of each chunk
//              with 16-byte cp.async copies (32 lanes generate addresses in
//              parallel; many small TMA row gathers were issue-bound) straight
//              into 128-byte-swizzled K-major UMMA tiles, in a ring of three
//              128-row slots (warp w copies rows 64w..64w+63 of a slot); they
//              also prefetch the rows of the fill two steps ahead into L2;
//   warp 2     TMEM owner; its lane 0 issues the S UMMAs, lane 0 of warp 3
//              the PV UMMAs, each waiting on one barrier at a time;
//   warps 4-7  softmax + epilogue of the even steps, warps 8-11 of the odd
//              steps (one query row per thread), so that one step's softmax
//              overlaps the other step's UMMAs, loads and stores.
// Key lengths come from the S tile itself: the pair's rows are also its keys,
// so row r finds ||k||^2 of its own row on the diagonal (key 64 + r % 64) and
// publishes the key multiplier scale * log2(e) / ||k||; the rows of a unit's
// leading chunk (which no earlier step of this CTA saw) are measured directly
// from shared memory.  The softmax uses the Cauchy-Schwarz bound
// q.k / ||k|| <= ||q|| as its shift (one pass over S, P written back as it
// goes); a row whose sum would underflow under that shift has its S rebuilt
// from shared memory and is redone with its exact maximum.  O is normalised by
// the sum of the bf16 weights P holds, which 12 more UMMAs of P against a
// tile of ones leave beside O.  The per-round outputs are stored with an L2
// evict-first policy (written once, read once by the merge), so that the rows
// the slice's other rounds gather again stay in L2.
// Masks are compile-time bits: causal (key positions against the query's),
// bucket (each row's bucket lands with the row), and with the bucket mask the
// multi-round union correction (each row's bucket in every round, up to 8,
// lands with the row; each admissible logit is lowered by log2 of the number of
// rounds the pair shares).
// TMEM: two step buffers of 256 columns (S: 192 fp32, P: first 96, O: 96..96+D,
// row sums: 16 columns after O).
// Every wait is bounded; a timeout unwinds the CTA cleanly.
#pragma once

#include <cuda_fp16.h>

#include "tc_common.cuh"

namespace lsh {
namespace att_tc {

constexpr int kC = 64;         // chunk length served
constexpr int kRows = 128;     // query rows per step
constexpr int kSlots = 3;      // 128-row slots in the shared-memory ring
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBufCols = 256;  // one step buffer
constexpr uint32_t kOOff = 96;      // O columns inside a step buffer
// registers per thread after the launch's 168: warpgroup 0 (producers, issuers)
// gives up 64, the two softmax warpgroups take 24 each (128 x 64 >= 256 x 24)
constexpr uint32_t kLowRegs = 104, kSoftRegs = 192;
template <int D>
__host__ __device__ constexpr uint32_t lr_col() { return kOOff + D; }

// Compile-time masks of an instantiation (besides the self mask, a runtime flag).
constexpr int kMaskCausal = 1;  // a key after the query's original position is not admissible
constexpr int kMaskBucket = 2;  // a key in another bucket than the query's is not admissible
// (with kMaskBucket) each admissible logit is lowered by log N, N = the number of
// rounds (at most kUnionRounds) whose hash puts query and key in one bucket
constexpr int kMaskUnion = 4;
constexpr int kUnionRounds = 8;
// Union rows code bucket b of a round as the fp16 bit pattern 0x0400 + b: a normal, positive,
// finite half, and distinct buckets give distinct values, so an fp16 compare is an exact bucket
// compare and no subnormal flushing can merge two buckets.  Buckets from kUnionMaxBucket up have no
// code; rounds that do not exist are -1.0 in a key's row and -2.0 in a query's, so they never agree.
constexpr int kUnionMaxBucket = 0x7C00 - 0x0400;  // 30720: 0x7C00 is +inf
constexpr uint16_t kUnionKeyNone = 0xBC00;        // -1.0
constexpr uint16_t kUnionQueryNone = 0xC000;      // -2.0

template <int D>
struct Layout {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kHalfBytes = kRows * 128;          // 128 rows x 64 bf16
  static constexpr uint32_t kSlotBytes = kHalves * kHalfBytes; // one tensor, one slot
  static constexpr uint32_t kQK = 0;
  static constexpr uint32_t kV = kSlots * kSlotBytes;
  static constexpr uint32_t kOnes = 2 * kSlots * kSlotBytes;        // 16 x 128 B of bf16 1.0 (row sums)
  static constexpr uint32_t kPerm = kOnes + 16 * 128;               // int32 [kSlots][128]
  static constexpr uint32_t kColMul = kPerm + kSlots * kRows * 4;   // float [kSlots][128]
  static constexpr uint32_t kBk = kColMul + kSlots * kRows * 4;     // int32 [kSlots][128] (bucket mask)
  // uint4 [kSlots][128]: every round's bucket of each row as 8 fp16 codes (union correction)
  static constexpr uint32_t kBkAll = kBk + kSlots * kRows * 4;
  static constexpr uint32_t kBar = kBkAll + kSlots * kRows * 16;
  // full[3] empty[3] cm_full[3] s_full[2] p_ready[2] o_full[2] buf_empty[2] done
  static constexpr int kNumBars = 18;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;   // tmem base, abort flag
  static constexpr uint32_t kBytes = kMisc + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;         // slack for 1024-byte alignment
};

struct Params {
  const int32_t* perm;   // [segs][L]
  const int32_t* buckets;  // [segs][L] by original position (bucket mask only)
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
  int sorted_input;      // rows are [seg][slot] of the sorted copies instead of [bh][pos]
  const uint8_t* qk;     // row sources (qk / v, or their sorted copies)
  const uint8_t* v;
  int out_v8;            // output rows 32-byte aligned: 32-byte stores
  // union correction: [bh][L] each token's bucket in every round of its (b, h) slice as 8 fp16 codes
  // (see kUnionMaxBucket), 16 bytes per token, one copy per row
  const uint4* bk_rows;
};

// Packs the union correction's per-token rows from buckets [bh][n_rounds][L]: one thread per token,
// 8 fp16 codes (round r in halfword r).  A bucket outside [0, kUnionMaxBucket) records
// LSH_ERR_UNSUPPORTED in the device status word and is coded as a NaN, which agrees with nothing.
__global__ void union_rows_kernel(const int32_t* __restrict__ buckets, long long n_tok, int n_rounds, int L,
                                  uint4* __restrict__ rows) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_tok) return;
  const long long bh = t / L, pos = t - bh * L;
  uint32_t code[kUnionRounds];
#pragma unroll
  for (int r = 0; r < kUnionRounds; ++r) {
    code[r] = kUnionKeyNone;
    if (r < n_rounds) {
      const int b = buckets[(bh * n_rounds + r) * L + pos];
      if (b >= 0 && b < kUnionMaxBucket) {
        code[r] = 0x0400u + (uint32_t)b;
      } else {
        record_error(LSH_ERR_UNSUPPORTED);
        code[r] = 0x7E00u;
      }
    }
  }
  rows[t] = make_uint4(code[0] | (code[1] << 16), code[2] | (code[3] << 16), code[4] | (code[5] << 16),
                       code[6] | (code[7] << 16));
}

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Warp-uniform bounded wait: every lane acquires the phase itself, lane 0
// decides on abort / timeout so that the warp leaves together.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  bool done = tc::mbar_try_wait(bar, parity);
  if (__all_sync(0xffffffffu, done)) return true;
  const unsigned long long t0 = tc::globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (!done) done = tc::mbar_try_wait_sleep(bar, parity, 20000u);
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

// Single-thread bounded wait for an UMMA issuer (the barrier wait's own short
// suspend; a longer suspend-time hint woke the issuers late): gives up on
// abort or after kWaitNs.
__device__ __forceinline__ bool issuer_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = tc::globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((i & 7u) == 0) {
      if (*abort_flag) return false;
      if (tc::globaltimer() - t0 > tc::kWaitNs) {
        *abort_flag = 1;
        record_error(LSH_ERR_TIMEOUT);
        return false;
      }
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

// Walks this CTA's steps in order.  A work unit is a run of consecutive steps
// of one (b, h, round) segment; each unit starts with one fill holding the
// chunk before its first pair, then one fill per step.  f is the fill index of
// the step's own pair; the previous chunk is always in fill f - 1.
struct StepIter {
  long long u;
  long long seg;
  int j, j1;
  uint32_t f;   // fill of the step's pair
  uint32_t t;   // step counter of this CTA
  bool valid;

  __device__ __forceinline__ void load_unit(const Params& p) {
    valid = u < p.n_units;
    if (!valid) return;
    seg = u / p.units_per_seg;
    j = (int)(u - seg * p.units_per_seg) * p.run;
    j1 = min(j + p.run, p.n_steps);
  }
  __device__ __forceinline__ void init(const Params& p) {
    u = blockIdx.x;
    f = 1;
    t = 0;
    load_unit(p);
  }
  __device__ __forceinline__ bool last_of_unit() const { return j + 1 >= j1; }
  __device__ __forceinline__ void advance(const Params& p) {
    ++t;
    if (j + 1 < j1) {
      ++j;
      ++f;
    } else {
      u += gridDim.x;
      f += 2;  // the next unit's leading fill, then its first pair
      load_unit(p);
    }
  }
};

// One fill of the slot ring: `nrows` rows (64 or 128) starting at local row
// `row0`; local rows [row0, row0+64) hold chunk cA, [row0+64, row0+128) chunk cB.
struct Fill {
  long long seg;
  int row0, nrows, cA, cB;
};

// Walks the fills of this CTA in order: per unit one leading fill (the chunk
// before the unit's first pair; chunk 0 again at a segment start, masked
// later) and then one fill per step (odd tail: the last chunk repeated, rows
// unused).
struct FillIter {
  long long u;
  int j, j0, j1;
  bool valid;
  __device__ __forceinline__ void load_unit(const Params& p) {
    valid = u < p.n_units;
    if (!valid) return;
    const long long seg = u / p.units_per_seg;
    j0 = (int)(u - seg * p.units_per_seg) * p.run;
    j1 = min(j0 + p.run, p.n_steps);
    j = j0 - 1;
  }
  __device__ __forceinline__ void init(const Params& p) {
    u = blockIdx.x;
    load_unit(p);
  }
  __device__ __forceinline__ Fill get(const Params& p) const {
    Fill f;
    f.seg = u / p.units_per_seg;
    if (j < j0) {
      f.row0 = 64;
      f.nrows = 64;
      f.cA = f.cB = j0 > 0 ? 2 * j0 - 1 : 0;
    } else {
      f.row0 = 0;
      f.nrows = 128;
      f.cA = 2 * j;
      f.cB = (2 * j + 1 < p.n_chunks) ? 2 * j + 1 : 2 * j;
    }
    return f;
  }
  __device__ __forceinline__ void advance(const Params& p) {
    if (j + 1 < j1) {
      ++j;
    } else {
      u += gridDim.x;
      load_unit(p);
    }
  }
};

// Original positions of this lane's two rows of the producer warp's half of a
// fill (global loads, issued one fill ahead so that their latency hides behind
// the slot wait).  Producer warp pw owns local rows [64 pw, 64 pw + 64).
__device__ __forceinline__ void fill_positions(const Params& p, const Fill& f, int pw, int (&pos)[2]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int i = 64 * pw + 32 * k + lane;  // local row of the slot
    pos[k] = 0;
    if (i >= f.row0 && i < f.row0 + f.nrows) {
      const int chunk = (i - f.row0) < 64 ? f.cA : f.cB;
      pos[k] = p.perm[f.seg * p.L + chunk * kC + (i & 63)];
    }
  }
}

// Gathers the producer warp's rows of a fill into slot `slot` with 16-byte
// cp.async copies: row r of a 128 x 64-element half tile sits at r * 128 bytes
// and its 16-byte piece c at ((c ^ (r % 8)) * 16), the 128-byte swizzle the
// UMMA descriptors expect.  Every producer lane then arrives on `full_bar`
// when its copies have landed.
template <int D, bool BUCKET, bool UNION>
__device__ __forceinline__ void producer_fill(const Params& p, uint8_t* smem, uint64_t* full_bar, int slot,
                                              const Fill& f, int pw, const int (&pos)[2]) {
  using Lay = Layout<D>;
  constexpr int kPieces = D / 8;            // 16-byte pieces per row
  constexpr int kRowsPerInst = 32 / kPieces;
  const int lane = threadIdx.x & 31;
  int32_t* perm_s = reinterpret_cast<int32_t*>(smem + Lay::kPerm) + slot * kRows;
  const int base = 64 * pw;
  const bool mine = base >= f.row0 && base < f.row0 + f.nrows;  // the fill covers this warp's rows
  if (mine) {
    long long grow[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = base + 32 * k + lane;
      const int chunk = (i - f.row0) < 64 ? f.cA : f.cB;
      perm_s[i] = pos[k];
      if (BUCKET)  // the row's bucket lands with the row (same cp.async group, same barrier)
        tc::cp_async4(tc::smem_u32(smem + Lay::kBk) + (slot * kRows + i) * 4, p.buckets + f.seg * p.L + pos[k]);
      if (UNION)  // the row's bucket in every round of its (b, h) slice: one 16-byte packed row
        tc::cp_async16(tc::smem_u32(smem + Lay::kBkAll) + (slot * kRows + i) * 16,
                       p.bk_rows + (f.seg / p.n_rounds) * p.L + pos[k]);
      grow[k] = p.sorted_input ? f.seg * p.L + chunk * kC + (i & 63) : (f.seg / p.n_rounds) * p.L + pos[k];
    }
    const uint32_t qk_dst = tc::smem_u32(smem + Lay::kQK + slot * Lay::kSlotBytes);
    const uint32_t v_dst = tc::smem_u32(smem + Lay::kV + slot * Lay::kSlotBytes);
    const int c = lane % kPieces;
#pragma unroll 4
    for (int it = 0; it < 64 / kRowsPerInst; ++it) {
      const int rl = it * kRowsPerInst + lane / kPieces;  // row within the warp's 64
      const long long g = __shfl_sync(0xffffffffu, rl < 32 ? grow[0] : grow[1], rl & 31);
      const int r = base + rl;
      const uint32_t off = (c >> 3) * Lay::kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
      tc::cp_async16(qk_dst + off, p.qk + (g * D + c * 8) * 2);
      tc::cp_async16(v_dst + off, p.v + (g * D + c * 8) * 2);
    }
  }
  tc::cp_async_arrive(full_bar);
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

// Reinterprets two packed fp16 codes.
__device__ __forceinline__ __half2 u32_half2(uint32_t w) {
  __half2 h;
  memcpy(&h, &w, 4);
  return h;
}

// The union correction of one key: log2 of the number of rounds whose buckets of query and key
// agree (`ku`: the key's row of 8 fp16 codes, `qu`: the query's, with the query-side code for
// rounds that do not exist).  Four packed compares give 1.0 per agreeing round; a key that shares
// no round is masked by the bucket test, and its count is taken as 1.
__device__ __forceinline__ float union_log2(const uint4* ku, const __half2 (&qu)[4]) {
  const uint4 a = *ku;
  __half2 c = __heq2(u32_half2(a.x), qu[0]);
  c = __hadd2(c, __heq2(u32_half2(a.y), qu[1]));
  c = __hadd2(c, __heq2(u32_half2(a.z), qu[2]));
  c = __hadd2(c, __heq2(u32_half2(a.w), qu[3]));
  const float n = __half2float(__hadd(__low2half(c), __high2half(c)));
  return __log2f(fmaxf(n, 1.f));
}

// A query row's codes for union_log2: its own row, rounds from n_rounds on replaced by the query-side
// code.
__device__ __forceinline__ void union_query(const uint4 row, int n_rounds, __half2 (&qu)[4]) {
  const uint32_t w[4] = {row.x, row.y, row.z, row.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t lo = 2 * k < n_rounds ? (w[k] & 0xffffu) : kUnionQueryNone;
    const uint32_t hi = 2 * k + 1 < n_rounds ? (w[k] >> 16) : kUnionQueryNone;
    qu[k] = u32_half2(lo | (hi << 16));
  }
}

template <int D, int MASK>
__device__ __forceinline__ void softmax_group(uint32_t sbuf, uint32_t pcol, int g, const uint32_t (&cur)[32],
                                              const float* cm, const int32_t* kp, const int32_t* kb, bool dead,
                                              bool self_grp, int lane, float m, float& l, int qpos, int qb,
                                              int& others, const uint4* ku, const __half2 (&qu)[4]) {
  constexpr bool CAUSAL = (MASK & kMaskCausal) != 0, BUCKET = (MASK & kMaskBucket) != 0;
  constexpr bool UNION = (MASK & kMaskUnion) != 0;
  // key multipliers (and positions, buckets) as 16-byte loads: each group's 32 values start on a
  // 16-byte boundary
  const float4* cm4 = reinterpret_cast<const float4*>(cm);
  const int4* kp4 = reinterpret_cast<const int4*>(kp);
  const int4* kb4 = reinterpret_cast<const int4*>(kb);
  uint32_t w16[16];
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float4 c4 = cm4[e >> 2];
    // shifted logits in the log2 domain, S * colmul - m as one FMA
    float v0 = fmaf(__uint_as_float(cur[e]), (e & 2) ? c4.z : c4.x, -m);
    float v1 = fmaf(__uint_as_float(cur[e + 1]), (e & 2) ? c4.w : c4.y, -m);
    if (CAUSAL || BUCKET) {  // keys are distinct tokens: position == qpos only for self
      bool c0 = true, c1 = true;  // counted: admissible and (CAUSAL) not self
      if (CAUSAL) {
        const int4 k4 = kp4[e >> 2];
        const int p0 = (e & 2) ? k4.z : k4.x, p1 = (e & 2) ? k4.w : k4.y;
        if (p0 > qpos) v0 = -INFINITY;
        if (p1 > qpos) v1 = -INFINITY;
        c0 = p0 < qpos;
        c1 = p1 < qpos;
      }
      if (BUCKET) {
        const int4 b4 = kb4[e >> 2];
        const int b0 = (e & 2) ? b4.z : b4.x, b1 = (e & 2) ? b4.w : b4.y;
        if (b0 != qb) v0 = -INFINITY;
        if (b1 != qb) v1 = -INFINITY;
        c0 = c0 && b0 == qb;
        c1 = c1 && b1 == qb;
      }
      if (!dead) others += (int)c0 + (int)c1;
    }
    if (UNION) {  // lower each logit by log2 of the rounds the pair shares
      v0 -= union_log2(ku + e, qu);
      v1 -= union_log2(ku + e + 1, qu);
    }
    if (self_grp) {
      if (e == lane) v0 = -INFINITY;
      if (e + 1 == lane) v1 = -INFINITY;
    }
    const float a = dead ? 0.f : tc::ex2_approx(v0);
    const float c = dead ? 0.f : tc::ex2_approx(v1);
    l += a + c;
    w16[e >> 1] = tc::pack_bf16x2(a, c);
  }
  tc::tmem_st16(sbuf + pcol + 16 * g, w16);
}

// One pass of the softmax over a row's 128 keys, four groups of 32 S columns
// (the next group's TMEM load in flight while the current one is processed): w = 2^(S * colmul - m) in fp32 (self masked, a missing previous chunk
// dead, with CAUSAL a key after the query's original position masked, with
// BUCKET a key outside the query's bucket masked), l += w, and the weights go
// to P as bf16 pairs right away: P's group g lands on S columns whose values
// this row has already consumed.  With MASK bits, `others` counts the
// admissible keys (CAUSAL: the earlier ones; BUCKET alone: those of the
// query's bucket, self included).
template <int D, int MASK>
__device__ __forceinline__ void softmax_pass(uint32_t sbuf, uint32_t scol, uint32_t pcol, const float* cm_lo,
                                             const float* cm_hi, int g_first, int g_self, int lane, int self_mask,
                                             float m, float& l, const int32_t* kp_lo, const int32_t* kp_hi,
                                             int qpos, const int32_t* kb_lo, const int32_t* kb_hi, int qb,
                                             int& others, const uint4* ku_lo, const uint4* ku_hi,
                                             const __half2 (&qu)[4]) {
  uint32_t ra[32], rb[32];
  tc::tmem_ld32(sbuf + scol, ra);
  tc::tmem_wait_ld_regs(ra);
#pragma unroll
  for (int h = 0; h < 2; ++h) {  // keys [64 h, 64 h + 64): groups 2h (in ra) and 2h + 1
    const float* cm = h ? cm_hi : cm_lo;
    const int32_t* kp = h ? kp_hi : kp_lo;
    const int32_t* kb = h ? kb_hi : kb_lo;
    const uint4* ku = h ? ku_hi : ku_lo;
    const bool dead = 2 * h < g_first;  // g_first is 0 or 2: both groups of the first half
    tc::tmem_ld32(sbuf + scol + 64 * h + 32, rb);
    softmax_group<D, MASK>(sbuf, pcol, 2 * h, ra, cm, kp, kb, dead, self_mask && 2 * h == g_self, lane, m, l,
                           qpos, qb, others, ku, qu);
    tc::tmem_wait_ld_regs(rb);
    if (h == 0) tc::tmem_ld32(sbuf + scol + 64, ra);
    softmax_group<D, MASK>(sbuf, pcol, 2 * h + 1, rb, cm + 32, kp + 32, kb + 32, dead,
                           self_mask && 2 * h + 1 == g_self, lane, m, l, qpos, qb, others,
                           ku + 32, qu);
    if (h == 0) tc::tmem_wait_ld_regs(ra);
  }
}

// Rows with no admissible key but themselves (causal: no earlier key; bucket:
// alone in their bucket inside the window) see only themselves: their P becomes
// one-hot at the own key (bf16 1.0 at element `lane` of the self group) and
// their weight sum 1 (the shift m is their own logit; under the union
// correction the self pair shares every round, so its weight is 1 / n_rounds).
// The whole warp rewrites the self group, the other rows with the words they
// already had (read back from TMEM).  `others` counts self too when only the
// bucket mask is on.
template <int MASK>
__device__ __forceinline__ void self_only_fixup(uint32_t sbuf, uint32_t pcol, int g_self, int lane, int others,
                                                float& l, float self_weight) {
  const bool only = (MASK & kMaskCausal) ? others == 0 : others <= 1;
  if (!__any_sync(0xffffffffu, only)) return;
  uint32_t w16[16];
  tc::tmem_wait_st();
  tc::tmem_ld16_wait(sbuf + pcol + 16 * g_self, w16);
#pragma unroll
  for (int k = 0; k < 16; ++k)
    if (only) w16[k] = k == (lane >> 1) ? ((lane & 1) ? 0x3F800000u : 0x00003F80u) : 0u;
  tc::tmem_st16(sbuf + pcol + 16 * g_self, w16);
  if (only) l = self_weight;
}

// Exact maximum of a row's scaled logits (self excluded while it has other keys;
// with MASK bits, keys after the query's position / outside its bucket excluded).
template <int MASK>
__device__ __noinline__ float exact_row_max(uint32_t sbuf, uint32_t scol, const float* cm_lo, const float* cm_hi,
                                               int g_first, int g_self, int lane, int self_mask,
                                               const int32_t* kp_lo, const int32_t* kp_hi, int qpos,
                                               const int32_t* kb_lo, const int32_t* kb_hi, int qb,
                                               const uint4* ku_lo, const uint4* ku_hi,
                                               const __half2 (&qu)[4]) {
  constexpr bool CAUSAL = (MASK & kMaskCausal) != 0, BUCKET = (MASK & kMaskBucket) != 0;
  constexpr bool UNION = (MASK & kMaskUnion) != 0;
  float m = -INFINITY;
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    uint32_t raw[32];
    tc::tmem_ld32(sbuf + scol + 32 * g, raw);
    tc::tmem_wait_ld_regs(raw);
    if (g < g_first) continue;
    const float* cm = g < 2 ? cm_lo + 32 * g : cm_hi + 32 * (g - 2);
    const int32_t* kp = g < 2 ? kp_lo + 32 * g : kp_hi + 32 * (g - 2);
    const int32_t* kb = g < 2 ? kb_lo + 32 * g : kb_hi + 32 * (g - 2);
    const uint4* ku = g < 2 ? ku_lo + 32 * g : ku_hi + 32 * (g - 2);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float v = __uint_as_float(raw[e]) * cm[e];
      if (UNION) v -= union_log2(ku + e, qu);
      if (CAUSAL && kp[e] > qpos) v = -INFINITY;
      if (BUCKET && kb[e] != qb) v = -INFINITY;
      if (g == g_self && self_mask && e == lane) v = -INFINITY;
      m = fmaxf(m, v);
    }
  }
  return m;
}

// Rebuilds the row's 128 S values (q . k, fp32) in TMEM from the QK tiles in
// shared memory: row r of the pair slot against keys [prev chunk rows 64..127,
// pair rows 0..63] (rows 0..63) or [pair rows 0..127] (rows 64..127).  Only
// the rare underflow path runs this.
template <int D>
__device__ __noinline__ void restore_s(const uint8_t* smem, uint32_t sbuf, uint32_t scol, int sp, int sc, int r,
                                       bool low) {
  using Lay = Layout<D>;
  const uint8_t* qs = smem + Lay::kQK + sc * Lay::kSlotBytes;
  const uint8_t* ps = smem + Lay::kQK + sp * Lay::kSlotBytes;
  tc::tmem_wait_st();  // P stores of the first pass land before S is rewritten
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    uint32_t out[32];
#pragma unroll 1
    for (int e = 0; e < 32; ++e) {
      const int k = 32 * g + e;  // key of the row's window
      const uint8_t* kt = low ? (k < 64 ? ps : qs) : qs;
      const int kr = low ? (k < 64 ? 64 + k : k - 64) : k;
      float acc = 0.f;
#pragma unroll 1
      for (int h = 0; h < Lay::kHalves; ++h) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float x[8], y[8];
          load8(reinterpret_cast<const __nv_bfloat16*>(qs + h * Lay::kHalfBytes + r * 128 + ((c ^ (r & 7)) << 4)), x);
          load8(reinterpret_cast<const __nv_bfloat16*>(kt + h * Lay::kHalfBytes + kr * 128 + ((c ^ (kr & 7)) << 4)), y);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc = fmaf(x[i], y[i], acc);
        }
      }
      out[e] = __float_as_uint(acc);
    }
    tc::tmem_st32(sbuf + scol + 32 * g, out);
  }
  tc::tmem_wait_st();
}

// 32 output values of a row (O columns times 1 / sum of the weights) with 32-byte
// stores (the row is 32-byte aligned) under the L2 policy `pol`.
__device__ __forceinline__ void store_o32(__nv_bfloat16* dst, const uint32_t (&raw)[32], float inv_l, uint64_t pol) {
#pragma unroll
  for (int e = 0; e < 32; e += 16) {  // 32 bf16 = two 32-byte stores
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k] = tc::pack_bf16x2(__uint_as_float(raw[e + 2 * k]) * inv_l, __uint_as_float(raw[e + 2 * k + 1]) * inv_l);
    tc::st_global_v8_hint(dst + e, w, pol);
  }
}
__device__ __forceinline__ void store_o32(float* dst, const uint32_t (&raw)[32], float inv_l, uint64_t pol) {
#pragma unroll
  for (int e = 0; e < 32; e += 8) {  // 32 floats = four 32-byte stores
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) w[k] = __float_as_uint(__uint_as_float(raw[e + k]) * inv_l);
    tc::st_global_v8_hint(dst + e, w, pol);
  }
}

// The epilogue for output rows that are only 16-byte aligned (16-byte stores),
// kept out of line: the aligned case is the one the warps run.
template <int D, typename TO>
__device__ __noinline__ void epilogue_plain(uint32_t sbuf, TO* dst, float inv_l, bool valid, uint64_t* buf_empty) {
#pragma unroll 1
  for (int g = 0; g < D / 32; ++g) {
    uint32_t raw[32];
    tc::tmem_ld32(sbuf + kOOff + 32 * g, raw);
    tc::tmem_wait_ld_regs(raw);
    if (g == D / 32 - 1) {
      tc::tc_fence_before();
      tc::mbar_arrive(buf_empty);
    }
    if (valid) {
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        float y[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = __uint_as_float(raw[e + k]) * inv_l;
        store8(dst + 32 * g + e, y);
      }
    }
  }
}

template <int D, typename TO, int MASK>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(const Params p) {
  using Lay = Layout<D>;
  constexpr bool MASKED = MASK != 0;  // a self-only fix-up may be needed
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte-aligned base as an offset from the shared array itself (not an integer
  // cast), so that every access through it stays a shared-memory access
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* full = bars;            // [3] slot filled (64 producer lanes' copies landed)
  uint64_t* empty = bars + 3;       // [3] slot released by the UMMAs
  uint64_t* cm_full = bars + 6;     // [3] key multipliers of the slot's fill written (128 arrivals)
  uint64_t* s_full = bars + 9;      // [2] S of the step buffer computed
  uint64_t* p_ready = bars + 11;    // [2] P written (128 arrivals)
  uint64_t* o_full = bars + 13;     // [2] O computed
  uint64_t* buf_empty = bars + 15;  // [2] O read (128 arrivals)
  uint64_t* done_bar = bars + 17;   // all UMMAs retired
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);
  float* colmul = reinterpret_cast<float*>(smem + Lay::kColMul);
  const int32_t* perm_s = reinterpret_cast<const int32_t*>(smem + Lay::kPerm);
  const int32_t* bk_s = reinterpret_cast<const int32_t*>(smem + Lay::kBk);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      tc::mbar_init(&full[i], 64);
      tc::mbar_init(&empty[i], 1);
      tc::mbar_init(&cm_full[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&s_full[i], 1);
      tc::mbar_init(&p_ready[i], 128);
      tc::mbar_init(&o_full[i], 1);
      tc::mbar_init(&buf_empty[i], 128);
    }
    tc::mbar_init(done_bar, 2);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  {
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + Lay::kOnes);
    for (int i = threadIdx.x; i < 16 * 128 / 4; i += kThreads) ones[i] = 0x3F803F80u;  // two bf16 1.0
    tc::fence_proxy_async_smem();
  }
  if (warp == 2) tc::tmem_alloc(tmem_holder, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < 4) {
    // warpgroup 0 (producers and UMMA issuers) hands registers to the softmax
    // warpgroups; every warp of a warpgroup executes the same setmaxnreg
    setmaxnreg_dec<kLowRegs>();
    if (warp < 2) {
      // ------------------------------------------------------------ producers
      // Fills F (gathered now), F+1 (positions loaded), F+2 (rows warmed in L2 with
      // per-line prefetches now; positions loaded one iteration earlier), F+3
      // (positions loading).  The gathers are latency-bound and shared memory holds
      // one fill in flight, so rows that reach L2 early shorten the next gathers.
      const int pw = warp;
      uint32_t f = 0;
      FillIter it0, it1, it2, it3;
      it0.init(p);
      it1 = it0;
      if (it1.valid) it1.advance(p);
      it2 = it1;
      if (it2.valid) it2.advance(p);
      it3 = it2;
      if (it3.valid) it3.advance(p);
      int pos0[2] = {0, 0}, pos1[2] = {0, 0}, pos2[2] = {0, 0};
      if (it0.valid) fill_positions(p, it0.get(p), pw, pos0);
      if (it1.valid) fill_positions(p, it1.get(p), pw, pos1);
      if (it2.valid) fill_positions(p, it2.get(p), pw, pos2);
      while (it0.valid) {
        int pos3[2] = {0, 0};
        if (it3.valid) fill_positions(p, it3.get(p), pw, pos3);
        if (it2.valid) {
          const Fill pf = it2.get(p);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int i = 64 * pw + 32 * k + lane;
            if (i >= pf.row0 && i < pf.row0 + pf.nrows) {
              const int chunk = (i - pf.row0) < 64 ? pf.cA : pf.cB;
              const long long g = p.sorted_input ? pf.seg * p.L + chunk * kC + (i & 63)
                                                 : (pf.seg / p.n_rounds) * p.L + pos2[k];
#pragma unroll
              for (int ln = 0; ln < D * 2; ln += 128) {
                tc::prefetch_l2_line(p.qk + g * D * 2 + ln);
                tc::prefetch_l2_line(p.v + g * D * 2 + ln);
              }
            }
          }
        }
        const Fill cur = it0.get(p);
        const int slot = f % kSlots;
        if (!warp_wait(&empty[slot], ((f / kSlots) & 1) ^ 1, abort_flag)) break;
        producer_fill<D, (MASK & kMaskBucket) != 0, (MASK & kMaskUnion) != 0>(p, smem, &full[slot], slot, cur, pw,
                                                                                 pos0);
        ++f;
        it0 = it1;
        it1 = it2;
        it2 = it3;
        if (it3.valid) it3.advance(p);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          pos0[k] = pos1[k];
          pos1[k] = pos2[k];
          pos2[k] = pos3[k];
        }
      }
      // never leave with copies in flight
      asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
      // ------------------------------------------------------------ UMMA issuers
      // warp 2 lane 0 issues the S UMMAs, warp 3 lane 0 the PV UMMAs; each waits
      // on one barrier at a time.  tcgen05.commit tracks the issuing thread's own
      // UMMAs.
      if (lane == 0) {
        const uint32_t qk0 = tc::smem_u32(smem + Lay::kQK);
        const uint32_t v0 = tc::smem_u32(smem + Lay::kV);
        StepIter it;
        it.init(p);
        if (warp == 2) {
          const uint32_t id_prev = tc::idesc_bf16_f32(128, 64, 0, 0);
          const uint32_t id_pair = tc::idesc_bf16_f32(128, 128, 0, 0);
          while (it.valid) {
            const uint32_t fp = it.f - 1, fc = it.f;
            if (!issuer_wait(&full[fp % kSlots], (fp / kSlots) & 1, abort_flag) ||
                !issuer_wait(&full[fc % kSlots], (fc / kSlots) & 1, abort_flag) ||
                !issuer_wait(&buf_empty[it.t & 1], ((it.t >> 1) & 1) ^ 1, abort_flag))
              break;
            tc::tc_fence_after();
            const uint32_t sbuf = tmem + (it.t & 1) * kBufCols;
            const uint32_t qk_c = qk0 + (fc % kSlots) * Lay::kSlotBytes;
            const uint32_t qk_p = qk0 + (fp % kSlots) * Lay::kSlotBytes + 64 * 128;  // rows 64..127
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (kk >> 2) * Lay::kHalfBytes + (kk & 3) * 32;
              const uint64_t a = tc::sdesc_sw128(qk_c + koff, 16, 1024);
              const uint64_t bp = tc::sdesc_sw128(qk_p + koff, 16, 1024);
              tc::umma_ss(sbuf, a, bp, id_prev, kk > 0);
              tc::umma_ss(sbuf + 64, a, a, id_pair, kk > 0);
            }
            tc::umma_commit(&s_full[it.t & 1]);
            it.advance(p);
          }
        } else {
          const uint32_t id_pv = tc::idesc_bf16_f32(128, D, 0, 1);
          const uint32_t id_lr = tc::idesc_bf16_f32(128, 16, 0, 1);
          const uint64_t ones_desc = tc::sdesc_sw128(tc::smem_u32(smem + Lay::kOnes), Lay::kHalfBytes, 1024);
          while (it.valid) {
            if (!issuer_wait(&p_ready[it.t & 1], (it.t >> 1) & 1, abort_flag)) break;
            tc::tc_fence_after();
            const uint32_t sbuf = tmem + (it.t & 1) * kBufCols;
            const uint32_t sp = (it.f - 1) % kSlots, sc = it.f % kSlots;
#pragma unroll
            for (int kk = 0; kk < 12; ++kk) {
              const uint32_t vrow = kk < 4 ? v0 + sp * Lay::kSlotBytes + (64 + 16 * kk) * 128
                                           : v0 + sc * Lay::kSlotBytes + (16 * (kk - 4)) * 128;
              const uint64_t b = tc::sdesc_sw128(vrow, Lay::kHalfBytes, 1024);
              tc::umma_ts(sbuf + kOOff, sbuf + kk * 8, b, id_pv, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 12; ++kk)  // every 16-key step reads the same 16 rows of ones
              tc::umma_ts(sbuf + lr_col<D>(), sbuf + kk * 8, ones_desc, id_lr, kk > 0);
            tc::umma_commit(&o_full[it.t & 1]);
            tc::umma_commit(&empty[sp]);
            if (it.last_of_unit()) tc::umma_commit(&empty[sc]);
            it.advance(p);
          }
        }
        tc::umma_commit(done_bar);
        drain_wait(done_bar, 0);
      }
      __syncwarp();
    }
  } else {
    setmaxnreg_inc<kSoftRegs>();
    // ------------------------------------------------------------ softmax + epilogue
    const int wg = (warp - 4) >> 2;      // 0: even steps, 1: odd steps
    const int q = warp & 3;              // TMEM lane quarter of this warp
    const int r = q * 32 + lane;         // query row of the step
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const bool low = q < 2;              // rows 0..63: keys [0, 128); rows 64..127: keys [64, 192)
    const int g_self = 2 + (q & 1);      // 32-key group of the row's own key; in it, element `lane`
    // per-round outputs are written once and read once by the merge: stored
    // evict-first, so that the rows the slice's rounds gather again stay in L2
    const uint64_t pol_out = tc::l2_evict_first();
    StepIter it;
    it.init(p);
    if (wg == 1) it.advance(p);
    bool ok = true;
    while (it.valid) {
      const uint32_t t = it.t, b = t & 1;
      const uint32_t fp = it.f - 1, fc = it.f;
      const int sp = fp % kSlots, sc = fc % kSlots;
      // the first step of a unit is the one whose previous chunk is the unit's leading fill
      const bool first = (it.j == (int)((it.u - it.seg * p.units_per_seg) * p.run));
      ok = warp_wait(&full[sc], (fc / kSlots) & 1, abort_flag) && warp_wait(&full[sp], (fp / kSlots) & 1, abort_flag) &&
           warp_wait(&s_full[b], (t >> 1) & 1, abort_flag);
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t sbuf = lane_base + tmem + b * kBufCols;
      const uint32_t scol = low ? 0 : 64;  // S column of the row's first key
      if (first) {  // the leading chunk's key multipliers, measured directly
        if (!low) colmul[sp * kRows + r] = row_colmul<D>(smem + Lay::kQK + sp * Lay::kSlotBytes, r, p.colscale);
        tc::mbar_arrive(&cm_full[sp]);
      }
      // own key multiplier from the diagonal of S (||k_r||^2 at key 64 + r % 64)
      float diag = 0.f;
      {
        uint32_t raw[32];
        tc::tmem_ld32(sbuf + scol + 32 * g_self, raw);
        tc::tmem_wait_ld_regs(raw);
#pragma unroll
        for (int e = 0; e < 32; ++e) diag = (e == lane) ? __uint_as_float(raw[e]) : diag;
      }
      const float cm_own = p.colscale / fmaxf(sqrtf(fmaxf(diag, 0.f)), 1e-12f);
      colmul[sc * kRows + r] = cm_own;
      tc::mbar_arrive(&cm_full[sc]);
      ok = warp_wait(&cm_full[sp], (fp / kSlots) & 1, abort_flag) &&
           warp_wait(&cm_full[sc], (fc / kSlots) & 1, abort_flag);
      if (!ok) break;
      const int chunk = 2 * it.j + (low ? 0 : 1);
      const bool valid = chunk < p.n_chunks;
      const int pos = perm_s[sc * kRows + r];
      const float* cm_lo = low ? colmul + sp * kRows + 64 : colmul + sc * kRows;  // keys 0..63 of the row
      const float* cm_hi = low ? colmul + sc * kRows : colmul + sc * kRows + 64;  // keys 64..127
      const int32_t* kp_lo = low ? perm_s + sp * kRows + 64 : perm_s + sc * kRows;  // their positions
      const int32_t* kp_hi = low ? perm_s + sc * kRows : perm_s + sc * kRows + 64;
      const int32_t* kb_lo = low ? bk_s + sp * kRows + 64 : bk_s + sc * kRows;      // their buckets
      const int32_t* kb_hi = low ? bk_s + sc * kRows : bk_s + sc * kRows + 64;
      const int qb = (MASK & kMaskBucket) ? bk_s[sc * kRows + r] : 0;
      // union correction: every round's bucket of the keys (per fill row) and of the query
      const uint4* bku = reinterpret_cast<const uint4*>(smem + Lay::kBkAll);
      const uint4* ku_lo = low ? bku + sp * kRows + 64 : bku + sc * kRows;
      const uint4* ku_hi = low ? bku + sc * kRows : bku + sc * kRows + 64;
      __half2 qu[4];
      union_query((MASK & kMaskUnion) ? bku[sc * kRows + r] : make_uint4(0u, 0u, 0u, 0u), p.n_rounds, qu);
      const float self_weight = (MASK & kMaskUnion) ? 1.f / (float)p.n_rounds : 1.f;
      int others = 0;
      const int g_first = (low && it.j == 0) ? 2 : 0;  // chunk 0 has no previous chunk
      // shift: ||q|| * scale * log2(e) bounds every logit of the row (log2 domain)
      const float m_cs = diag * cm_own;
      float m = m_cs;
      float l = 0.f;  // sum of the weights (log-sum-exp); O is normalised by the rounded weights' sum
      const uint32_t pcol = low ? 0 : 32;  // P column of the row's first key
#pragma unroll 1
      for (int attempt = 0;; ++attempt) {
        l = 0.f;
        others = 0;
        softmax_pass<D, MASK>(sbuf, scol, pcol, cm_lo, cm_hi, g_first, g_self, lane, p.self_mask, m, l, kp_lo,
                              kp_hi, pos, kb_lo, kb_hi, qb, others, ku_lo, ku_hi, qu);
        if (MASKED) self_only_fixup<MASK>(sbuf, pcol, g_self, lane, others, l, self_weight);
        if (attempt > 0 || !__any_sync(0xffffffffu, !(l > 1e-30f))) break;
        // the bound was too loose for some row of the warp (long query rows): S is
        // rebuilt in TMEM from the rows in shared memory (P has overwritten part of
        // it) and the warp's rows are redone with their exact maxima
        restore_s<D>(smem, sbuf, scol, sp, sc, r, low);
        m = exact_row_max<MASK>(sbuf, scol, cm_lo, cm_hi, g_first, g_self, lane, p.self_mask, kp_lo, kp_hi, pos,
                                kb_lo, kb_hi, qb, ku_lo, ku_hi, qu);
        if (MASKED && m == -INFINITY) m = m_cs;  // self-only row: its own logit is the shift
      }
      {
        uint32_t z[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) z[e] = 0u;
        tc::tmem_st32(sbuf + (low ? 64 : 0), z);
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(&p_ready[b]);
      // epilogue: O row -> original position
      ok = warp_wait(&o_full[b], (t >> 1) & 1, abort_flag);
      if (!ok) break;
      tc::tc_fence_after();
      // O = sum p~ v / sum p~ (p~ the bf16 weights in P): a convex combination of the values
      const float inv_l = 1.f / __uint_as_float(tc::tmem_ld1(sbuf + lr_col<D>()));
      TO* dst = reinterpret_cast<TO*>(p.out) + (it.seg * p.L + pos) * (long long)D;
      if (p.out_v8) {
#pragma unroll
        for (int g = 0; g < D / 32; ++g) {
          uint32_t raw[32];
          tc::tmem_ld32(sbuf + kOOff + 32 * g, raw);
          tc::tmem_wait_ld_regs(raw);
          if (g == D / 32 - 1) {
            tc::tc_fence_before();
            tc::mbar_arrive(&buf_empty[b]);
          }
          if (valid) store_o32(dst + 32 * g, raw, inv_l, pol_out);
        }
      } else {
        epilogue_plain<D, TO>(sbuf, dst, inv_l, valid, &buf_empty[b]);
      }
      if (valid) p.lse[it.seg * p.L + pos] = (m + __log2f(l)) * 0.6931471805599453f;
      it.advance(p);
      if (it.valid) it.advance(p);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace att_tc
}  // namespace lsh

// Backward of the chunk attention and the round merge on the 5th-generation
// tensor cores (tcgen05 + TMEM).
//
// Training through LSH attention recomputes from the stored hash (twgreatdaily
// ICLR 2020 Reformer article, section "1 LSH Attention"; Ultralytics glossary
// "Reformer", "Atencao LSH"): perm stays fixed.  With the rounds merged by their
// log-sum-exp, an admissible pair (i, j) of a round has the merged weight
// p~_ij = exp(z_ij - LSE_i), z_ij = scale (x_i . x_j) / ||x_j||, and the
// gradient of sum(dout * out) is
//     dz_ij = p~_ij (dout_i . v_j - dout_i . out_i)
//     dv_j += p~_ij dout_i
//     dx_i += scale dz_ij x_j / ||x_j||                        (query role)
//     dx_j += G_j - (x_j . G_j) x_j / ||x_j||^2,
//             G_j = scale sum_i dz_ij x_i / ||x_j||            (key role through the
//                                                              key normalisation)
// With Z_ij = scale dz_ij / ||x_j|| both roles are plain products:
// dQ = Z X (over the keys) and G = Z^T X (over the queries).
//
// Served case: bf16 rows and bf16 out / dout, D = 128, chunk 64, L a multiple
// of 128, the plain window with or without the self mask.  One launch per round
// (rounds in order: each adds into the fp32 gradients the previous ones left;
// the first one stores).  A fill is two consecutive sorted chunks (2t, 2t+1),
// 128 query rows; its key window is the three chunks 2t-1, 2t, 2t+1, taken one
// 64-key block at a time.  Per block b:
//   S_b  [128 x 64] = X_fill X_b^T      (TMEM, fp32)
//   dP_b [128 x 64] = dO_fill V_b^T
//   P~ = exp2(S s_j - LSE_i log2 e), Z = P~ (dP - Delta_i) scale / ||x_j||  (bf16,
//        shared memory, written by the softmax warps; rows outside the block's
//        window are never read)
//   dK^T, dV^T of the block's 64 keys  [128 (D) x 64] += X_fill^T Z, dO_fill^T P~
//   dQ^T of each query chunk that sees the block [128 x 64] += X_b^T Z^T
// All gradients are kept transposed (TMEM lane = feature d, column = token), so
// that a chunk's query-role and key-role sums land in the same columns: one
// TMEM region per chunk holds H = dQ + G and the dv sums, in a ring of three
// regions (chunk 2t+1 is finished by the next fill's first block).  The
// epilogue warps take a finished region: x_j . H_j (a reduction over the 128
// lanes) minus x_j . dQ_j (= sum_k Z_jk S_jk, summed by the softmax warps as
// they go) gives x_j . G_j for the key-normalisation term; the rows go to
// dqk / dv at the tokens' original positions (32 lanes cover 128 consecutive
// bytes of one row), stored by the first round and added in L2 by the later
// ones (fire-and-forget reductions: one writer per element and launch, so the
// sums do not depend on timing).
//
// Work units are runs of fills of one (b, h) segment.  A unit's first fill
// takes the chunk before it from a leading fill, whose key-role sums belong to
// the previous unit; a unit that ends before its segment does runs one more
// half fill (the next unit's first query chunk against its last chunk, key
// role only), so every token's rows have one writer per launch: no atomics,
// and reruns are bit-identical.
//
// Warp roles (512 threads, one CTA per SM; launched at 128 registers, warpgroup
// 0 gives 56 to the others with setmaxnreg: 72 / 144 / 144 / 152):
//   warps 0-1   producers: 16-byte cp.async row gathers (X, V, then dO) through
//               perm into 128-byte-swizzled tiles, two fill slots for X and V,
//               one dO tile (warp w its rows 64 w .., each half with its own
//               barriers, so the next fill's rows 0..63 load during block 2),
//               plus each row's LSE, Delta and length terms;
//   warps 2-3   UMMA issuers (lane 0): warp 2 the S and dP of each block, warp 3
//               the gradient products; warp 2 also owns the TMEM allocation;
//   warps 4-11  softmax: both warpgroups take every row (TMEM lane), keys
//               0-31 / 32-63 of each block;
//   warps 12-15 epilogue.
// TMEM (512 columns): S (64) and dP (64) of the current block, then three
// chunk regions of H (64) and dv (64).  Every wait is bounded; a timeout
// unwinds the CTA cleanly.
#pragma once

#include "attend_tc.cuh"

namespace lsh {
namespace bwd_tc {

constexpr int kC = 64;
constexpr int kRows = 128;
constexpr int kD = 128;
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
// TMEM: two S/dP buffers of 128 columns (S 64, dP 64), then two chunk regions of H (64) and dv (64)
constexpr uint32_t kSPCols = 128, kPOff = 64, kRegCol0 = 256, kRegCols = 128;

// mbarrier indices
struct Bars {
  static constexpr int kSlotFull = 0;   // [2] a fill's rows and tables landed (64 producer lanes)
  static constexpr int kSlotFree = 2;   // [2] a fill slot may be refilled
  static constexpr int kDoFull = 4;     // dO rows 0..63 landed (producer warp 0)
  static constexpr int kDoFree = 5;     // dO rows 0..63 read by their last UMMA
  static constexpr int kSpFull = 6;     // [2] S and dP of a block computed (buffer kb % 2)
  static constexpr int kSpFree = 8;     // [2] S and dP loaded by the softmax (256)
  static constexpr int kPzFull = 10;    // P~ and Z of a block written (256)
  static constexpr int kPzFree = 11;    // P~ and Z read by the block's UMMAs
  static constexpr int kHvDone = 12;    // [2] a chunk region finished
  static constexpr int kHvHFree = 14;   // [2][2] a region's H columns 0..31 / 32..63 read by the epilogue (128)
  static constexpr int kHvVFree = 18;   // [2] a region's dv columns read by the epilogue (128)
  static constexpr int kRFull = 20;     // [2] x . dQ partials of a fill written (256)
  static constexpr int kDone = 22;      // every UMMA retired (both issuers)
  static constexpr int kDoFull1 = 23;   // dO rows 64..127 landed (producer warp 1)
  static constexpr int kDoFree1 = 24;   // dO rows 64..127 read by their last UMMA
  static constexpr int kCount = 25;
};
// registers per thread after the launch's 128: 72 (producers, issuer), 144 (softmax), 152 (epilogue);
// 128 x (72 + 2 x 144 + 152) = 65536
constexpr uint32_t kLowRegs = 72, kSoftRegs = 144, kEpiRegs = 152;

struct Layout {
  static constexpr uint32_t kHalf = kRows * 128;       // 128 rows x 64 bf16
  static constexpr uint32_t kTile = 2 * kHalf;         // 128 rows x 128 bf16
  static constexpr uint32_t kQK = 0;                   // [2] X rows of a fill slot
  static constexpr uint32_t kV = 2 * kTile;            // [2] V rows
  static constexpr uint32_t kDO = 4 * kTile;           // dO rows of the current fill
  static constexpr uint32_t kP = 5 * kTile;            // P~ of one key block [128 x 64] bf16
  static constexpr uint32_t kZ = kP + kHalf;           // Z of one key block
  static constexpr uint32_t kAux = kZ + kHalf;         // float4 [2][128]: LSE log2 e, Delta, 1/||x||, kcorr
  static constexpr uint32_t kKinv = kAux + 2 * kRows * 16;  // float [2][128]: 1/||x|| (vector loads)
  static constexpr uint32_t kPerm = kKinv + 2 * kRows * 4;  // int32 [2][128]: original positions
  static constexpr uint32_t kR = kPerm + 2 * kRows * 4;     // float [2][2][128]: x_i . dQ_i partials
  static constexpr uint32_t kXH = kR + 2 * 2 * kRows * 4;   // float [4][32]: epilogue partial sums
  static constexpr uint32_t kStage = kXH + 4 * 32 * 4;      // float [4 warps][32 tokens][32 features]
  // masks: int32 [2][128]: the row's bucket in this round | (1 << 31) when its window leaves it alone
  static constexpr uint32_t kMaskRow = kStage + 4 * 32 * 32 * 4;
  static constexpr uint32_t kBar = kMaskRow + 2 * kRows * 4;
  static constexpr int kNumBars = Bars::kCount;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;  // tmem base, abort flag
  static constexpr uint32_t kBytes = kMisc + 16;
  // union correction only: uint4 [2][128], each row's bucket in every round as 8 fp16 codes (as in
  // the forward's union rows); read by 16-byte copies and loads, so 128-byte aligned
  static constexpr uint32_t kUnion = (kBytes + 127u) & ~127u;
  static constexpr uint32_t smem(bool with_union) {
    return (with_union ? kUnion + 2 * kRows * 16 : kBytes) + 1024;
  }
};

// 16-byte copies and vector accesses land on these regions; the whole layout fits one SM
static_assert(Layout::kAux % 16 == 0 && Layout::kKinv % 16 == 0 && Layout::kStage % 16 == 0 &&
                  Layout::kUnion % 16 == 0 && Layout::kBar % 8 == 0 && Layout::kP % 1024 == 0 &&
                  Layout::kZ % 1024 == 0 && Layout::kDO % 1024 == 0,
              "backward layout alignment");
static_assert(Layout::smem(true) <= 227 * 1024, "backward layout exceeds the shared memory of an SM");

struct Params {
  const uint8_t* qk;      // bf16 [bh][L][128]
  const uint8_t* v;
  const uint8_t* dout;
  const int32_t* perm;    // [bh][n_rounds][L]
  const float4* aux;      // [bh][L]: LSE log2 e, dout . out, 1/max(||x||, 1e-12), (||x|| >= 1e-12) / ||x||^2
  float* dqk;             // fp32 [bh][L][128]
  float* dv;
  int L;
  int n_rounds;
  int round;
  int n_fills;            // L / 128
  int run;                // fills per work unit
  int units_per_seg;
  long long n_units;
  int self_mask;
  float scale;
  int accumulate;         // 0: the first round stores, 1: later rounds add
  // masks (compile-time bits of the instantiation): [bh][n_rounds][L] by original position, the
  // token's bucket in the round (bucket mask) | (1 << 31) when its window leaves it alone
  const int32_t* mask_rows;
  const uint4* bk_rows;    // union: [bh][L] every round's bucket of each token as 8 fp16 codes
};

// Compile-time masks of a backward instantiation (as in the forward's attention).
constexpr int kMaskCausal = att_tc::kMaskCausal, kMaskBucket = att_tc::kMaskBucket, kMaskUnion = att_tc::kMaskUnion;

enum : int { kLead = 0, kFull = 1, kHalo = 2 };

// Walks this CTA's fills: per unit a leading fill (chunk 2 t0 - 1 in rows
// 64..127; nothing to copy at a segment start), the unit's fills t0 .. t1-1,
// and, when the segment goes on, the half fill t1 (chunk 2 t1 in rows 0..63).
struct FillIt {
  long long u, bh;
  int t, t0, t1, kind;
  bool valid;
  __device__ __forceinline__ void load_unit(const Params& p) {
    valid = u < p.n_units;
    if (!valid) return;
    bh = u / p.units_per_seg;
    t0 = (int)(u - bh * p.units_per_seg) * p.run;
    t1 = min(t0 + p.run, p.n_fills);
    t = t0;
    kind = kLead;
  }
  __device__ __forceinline__ void init(const Params& p) {
    u = blockIdx.x;
    load_unit(p);
  }
  __device__ __forceinline__ void advance(const Params& p) {
    if (kind == kLead) {
      kind = kFull;
    } else if (kind == kFull && t + 1 < t1) {
      ++t;
    } else if (kind == kFull && t1 < p.n_fills) {
      kind = kHalo;
      t = t1;
    } else {
      u += gridDim.x;
      load_unit(p);
    }
  }
  __device__ __forceinline__ bool has_prev() const { return t > 0; }
  // the key-role sums of chunk 2t-1 belong to this unit (not to the previous one)
  __device__ __forceinline__ bool owns_prev() const { return t > 0 && (kind == kHalo || t > t0); }
};

// Original positions of this producer lane's two rows of a fill (rows 64 pw + lane, +32).
__device__ __forceinline__ bool fill_rows(const Params& p, const FillIt& f, int pw, int (&pos)[2]) {
  const int lane = threadIdx.x & 31;
  // rows present: lead -> 64..127 (if t0 > 0); full -> 0..127; halo -> 0..63
  bool mine;
  int chunk;
  if (f.kind == kLead) {
    mine = pw == 1 && f.t0 > 0;
    chunk = 2 * f.t0 - 1;
  } else if (f.kind == kHalo) {
    mine = pw == 0;
    chunk = 2 * f.t;
  } else {
    mine = true;
    chunk = 2 * f.t + pw;
  }
  pos[0] = pos[1] = 0;
  if (mine) {
    const int32_t* pr = p.perm + (f.bh * p.n_rounds + p.round) * (long long)p.L + chunk * kC;
    pos[0] = pr[lane];
    pos[1] = pr[32 + lane];
  }
  return mine;
}

// Gathers 64 rows (local rows 64 pw ..) of each listed tensor into a 128-row
// swizzled tile: 16-byte piece c of row r at (c / 8) * kHalf + r * 128 +
// ((c % 8) ^ (r % 8)) * 16, the layout the UMMA descriptors expect.
__device__ __forceinline__ void gather64(uint32_t dst, const uint8_t* src, long long rowbase, int pw,
                                         const int (&pos)[2]) {
  const int lane = threadIdx.x & 31;
  const int c = lane & 15;
#pragma unroll 4
  for (int it = 0; it < 32; ++it) {
    const int rl = 2 * it + (lane >> 4);  // row within the warp's 64
    const int pr = __shfl_sync(0xffffffffu, rl < 32 ? pos[0] : pos[1], rl & 31);
    const int r = 64 * pw + rl;
    const uint32_t off = (c >> 3) * Layout::kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4);
    tc::cp_async16(dst + off, src + ((rowbase + pr) * kD + c * 8) * 2);
  }
}

// Barrier among `n` threads that also ANDs their predicates: a group decides together whether to go on.
__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.b32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((int)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void load4_bf16(const __nv_bfloat16* p, float (&o)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  o[0] = __low2float(a);
  o[1] = __high2float(a);
  o[2] = __low2float(b);
  o[3] = __high2float(b);
}

__device__ __forceinline__ void red_add_v4(float* p, float4 v) {  // 16-byte aligned
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

__device__ __forceinline__ uint32_t swz(int r, int c) {  // 16-byte piece c (0..7) of row r of a 64-wide tile
  return (uint32_t)(r * 128 + (((c ^ r) & 7) << 4));
}

// lane l of the result holds the sum over the warp's lanes of v[l]
__device__ __forceinline__ float transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool hi = (lane & o) != 0;
#pragma unroll
    for (int e = 0; e < o; ++e) {
      const float send = hi ? v[e] : v[e + o];
      const float keep = hi ? v[e + o] : v[e];
      v[e] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

// 16-feature step kk of a K-major operand (rows along M/N, 128 features, two 64-wide halves)
__device__ __forceinline__ uint64_t kdesc(uint32_t row0, int kk) {
  return tc::sdesc_sw128(row0 + (kk >> 2) * Layout::kHalf + (kk & 3) * 32, 16, 1024);
}
// MN-major operand whose K index is the tile row, starting at row r0 (a multiple of 16)
__device__ __forceinline__ uint64_t mdesc(uint32_t tile, int r0) {
  return tc::sdesc_sw128(tile + r0 * 128, Layout::kHalf, 1024);
}
// D (+)= A B^T over `steps` 16-wide K steps; A and B advance by a_step / b_step bytes per step
__device__ __forceinline__ void mma_run(uint32_t d, uint64_t a, uint32_t a_step, uint64_t b, uint32_t b_step,
                                        uint32_t idesc, int steps, bool acc) {
#pragma unroll 1
  for (int kk = 0; kk < steps; ++kk) {
    tc::umma_ss(d, a + (uint64_t)((kk * a_step) >> 4), b + (uint64_t)((kk * b_step) >> 4), idesc, acc || kk > 0);
  }
}

// S = X_fill X_b^T and dP = dO_fill V_b^T of one 64-key block (rows kx / kv of the X / V tiles)
// into the S/dP buffer at TMEM column sp
__device__ __forceinline__ void issue_sdp(uint32_t sp, uint32_t xs, uint32_t do0, uint32_t kx, uint32_t kv,
                                          uint64_t* sp_full) {
  const uint32_t id_s = tc::idesc_bf16_f32(128, 64, 0, 0);  // both K-major
#pragma unroll 1
  for (int kk = 0; kk < kD / 16; ++kk) {
    tc::umma_ss(sp, kdesc(xs, kk), kdesc(kx, kk), id_s, kk > 0);
    tc::umma_ss(sp + kPOff, kdesc(do0, kk), kdesc(kv, kk), id_s, kk > 0);
  }
  tc::umma_commit(sp_full);
}

// Lane 0 of warp 2: the S and dP UMMAs of every block, in fill order, into two alternating TMEM
// buffers; each waits until the softmax has loaded the block two before it from the same buffer.
__device__ __noinline__ void issuer_s(const Params& p, uint8_t* smem, uint32_t tmem, volatile int* abort_flag) {
  using Lay = Layout;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* slot_full = bars + Bars::kSlotFull;
  uint64_t* slot_free = bars + Bars::kSlotFree;
  uint64_t* do_full[2] = {bars + Bars::kDoFull, bars + Bars::kDoFull1};  // dO rows 0..63 / 64..127 landed
  uint64_t* sp_full = bars + Bars::kSpFull;
  uint64_t* sp_free = bars + Bars::kSpFree;
  const uint32_t qk0 = tc::smem_u32(smem + Lay::kQK), v0 = tc::smem_u32(smem + Lay::kV);
  const uint32_t do0 = tc::smem_u32(smem + Lay::kDO);
  FillIt f;
  f.init(p);
  uint32_t F = 0, nd = 0, nf = 0, kb = 0;  // fills, fills with dO rows 0..63, full fills, blocks
  bool ok = true;
  while (ok && f.valid) {
    const uint32_t s = F & 1, sp = (F + 1) & 1;
    if (f.kind == kLead) {
      ++F;
      f.advance(p);
      continue;
    }
    const bool full = f.kind == kFull, has_prev = f.has_prev();
    ok = att_tc::issuer_wait(&slot_full[s], (F >> 1) & 1, abort_flag) &&
         (!has_prev || att_tc::issuer_wait(&slot_full[sp], ((F - 1) >> 1) & 1, abort_flag));
    if (!ok) break;
    tc::tc_fence_after();
    if (full && f.t == f.t0 && !has_prev) tc::umma_commit(&slot_free[sp]);  // nothing of the leading fill is read
    const uint32_t xs = qk0 + s * Lay::kTile, vs = v0 + s * Lay::kTile;
    const uint32_t xp = qk0 + sp * Lay::kTile, vp = v0 + sp * Lay::kTile;
    // blocks: 0 = chunk 2t-1 (rows 64.. of the previous slot), 1 = chunk 2t, 2 = chunk 2t+1
    // the query rows' dO: block 0 needs rows 0..63 (its rows 64.. are not in its window), blocks 1
    // and 2 (full fills only) all 128.  Rows 64.. are handed over once per full fill and rows 0..63
    // once per fill, so that neither barrier can run two phases ahead of its waiter.
    bool top = false, bot = false;
    for (int b = has_prev ? 0 : 1; b <= (full ? 2 : 0); ++b) {
      ok = att_tc::issuer_wait(&sp_free[kb & 1], ((kb >> 1) & 1) ^ 1, abort_flag) &&
           (top || att_tc::issuer_wait(do_full[0], nd & 1, abort_flag)) &&
           (b == 0 || bot || att_tc::issuer_wait(do_full[1], nf & 1, abort_flag));
      if (!ok) break;
      top = true;
      bot = bot || b > 0;
      tc::tc_fence_after();
      const uint32_t kx = b == 0 ? xp + 64 * 128 : xs + (b == 2 ? 64 * 128 : 0);
      const uint32_t kv = b == 0 ? vp + 64 * 128 : vs + (b == 2 ? 64 * 128 : 0);
      issue_sdp(tmem + (kb & 1) * kSPCols, xs, do0, kx, kv, &sp_full[kb & 1]);
      ++kb;
    }
    ++nd;
    if (full) ++nf;
    ++F;
    f.advance(p);
  }
  uint64_t* done_bar = bars + Bars::kDone;
  tc::umma_commit(done_bar);
  att_tc::drain_wait(done_bar, 0);
}

// Lane 0 of warp 3: the gradient UMMAs of every block (dK^T, dV^T of its keys, dQ^T of the query
// chunks that see it), in fill order, each once the softmax has written the block's P~ and Z.
__device__ __noinline__ void issuer_hv(const Params& p, uint8_t* smem, uint32_t tmem, volatile int* abort_flag) {
  using Lay = Layout;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* slot_free = bars + Bars::kSlotFree;
  uint64_t* do_free[2] = {bars + Bars::kDoFree, bars + Bars::kDoFree1};  // dO rows 0..63 / 64..127 read
  uint64_t* pz_full = bars + Bars::kPzFull;
  uint64_t* pz_free = bars + Bars::kPzFree;
  uint64_t* hv_done = bars + Bars::kHvDone;
  uint64_t* hvh_free = bars + Bars::kHvHFree;
  uint64_t* hvv_free = bars + Bars::kHvVFree;
  const uint32_t qk0 = tc::smem_u32(smem + Lay::kQK);
  const uint32_t do0 = tc::smem_u32(smem + Lay::kDO);
  const uint32_t pt = tc::smem_u32(smem + Lay::kP), zt = tc::smem_u32(smem + Lay::kZ);
  const uint32_t id_kv = tc::idesc_bf16_f32(128, 64, 1, 1);  // dK^T, dV^T: both MN-major
  const uint32_t id_q = tc::idesc_bf16_f32(128, 64, 1, 0);   // dQ^T: A MN-major, B K-major
  const uint32_t id_q32 = tc::idesc_bf16_f32(128, 32, 1, 0); // dQ^T for 32 queries
  constexpr uint32_t kRowStep = 16 * 128;                    // 16 tile rows
  FillIt f;
  f.init(p);
  uint32_t F = 0, kb = 0, n = 0;  // fills, blocks, owned chunks
  bool ok = true;
  while (ok && f.valid) {
    const uint32_t s = F & 1, sp = (F + 1) & 1;
    if (f.kind == kLead) {
      ++F;
      f.advance(p);
      continue;
    }
    const bool full = f.kind == kFull, has_prev = f.has_prev(), owns_prev = f.owns_prev();
    const bool first = full && f.t == f.t0, seg_end = full && f.t == p.n_fills - 1;
    const uint32_t xs = qk0 + s * Lay::kTile, xp = qk0 + sp * Lay::kTile;
    // regions: chunk 2t-1 -> owned chunk n-1, 2t -> n, 2t+1 -> n+1, in a ring of two (chunk 2t+1 takes
    // the region of chunk 2t-1).  Before chunk c first writes H (or dv) the epilogue must have read
    // the H (dv) columns of chunk c-2: hvh_free / hvv_free[c % 2], parity ((c / 2) & 1) ^ 1.
    const uint32_t r0 = tmem + kRegCol0 + (n & 1) * kRegCols;        // chunk 2t
    const uint32_t r1 = tmem + kRegCol0 + ((n + 1) & 1) * kRegCols;  // chunk 2t+1, and chunk 2t-1 before it
    auto free_wait = [&](uint64_t* bar, uint32_t c) {  // dv columns of chunk c's region
      if (!att_tc::issuer_wait(&bar[c & 1], ((c >> 1) & 1) ^ 1, abort_flag)) return false;
      tc::tc_fence_after();
      return true;
    };
    auto free_wait_h = [&](uint32_t c, int half) {  // H columns 32 half .. of chunk c's region
      if (!att_tc::issuer_wait(&hvh_free[(c & 1) * 2 + half], ((c >> 1) & 1) ^ 1, abort_flag)) return false;
      tc::tc_fence_after();
      return true;
    };
    for (int b = has_prev ? 0 : 1; b <= (full ? 2 : 0); ++b) {
      ok = att_tc::issuer_wait(pz_full, kb & 1, abort_flag);
      if (!ok) break;
      tc::tc_fence_after();
      if (b == 0) {
        if (owns_prev) {  // key role of chunk 2t-1: queries of chunk 2t (rows 0..63)
          mma_run(r1, mdesc(xs, 0), kRowStep, mdesc(zt, 0), kRowStep, id_kv, 4, true);
          mma_run(r1 + 64, mdesc(do0, 0), kRowStep, mdesc(pt, 0), kRowStep, id_kv, 4, true);
        }
        if (full) {
          ok = free_wait_h(n, 0) && free_wait_h(n, 1);
          if (!ok) break;
          // dQ^T of chunk 2t from the keys of chunk 2t-1
          mma_run(r0, mdesc(xp + 64 * 128, 0), kRowStep, kdesc(zt, 0), 32, id_q, 4, false);
        }
        tc::umma_commit(pz_free);
        if (owns_prev) tc::umma_commit(&hv_done[(n + 1) & 1]);
        if (first) tc::umma_commit(&slot_free[sp]);  // the leading fill's slot (full fills: the epilogue)
      } else if (b == 1) {
        if (!has_prev) {
          ok = free_wait_h(n, 0) && free_wait_h(n, 1);
          if (!ok) break;
        }
        // key role of chunk 2t: all 128 queries
        mma_run(r0, mdesc(xs, 0), kRowStep, mdesc(zt, 0), kRowStep, id_kv, 8, has_prev);
        ok = free_wait(hvv_free, n);
        if (!ok) break;
        mma_run(r0 + 64, mdesc(do0, 0), kRowStep, mdesc(pt, 0), kRowStep, id_kv, 8, false);
        // dQ^T of chunk 2t from the keys of chunk 2t
        mma_run(r0, mdesc(xs, 0), kRowStep, kdesc(zt, 0), 32, id_q, 4, true);
        // dQ^T of chunk 2t+1 from the keys of chunk 2t, in two 32-query halves, each as soon as the
        // epilogue has read the same H columns of chunk 2t-1
        ok = free_wait_h(n + 1, 0);
        if (!ok) break;
        mma_run(r1, mdesc(xs, 0), kRowStep, kdesc(zt + 64 * 128, 0), 32, id_q32, 4, false);
        ok = free_wait_h(n + 1, 1);
        if (!ok) break;
        mma_run(r1 + 32, mdesc(xs, 0), kRowStep, kdesc(zt + 96 * 128, 0), 32, id_q32, 4, false);
        tc::umma_commit(pz_free);
        tc::umma_commit(&hv_done[n & 1]);
        tc::umma_commit(do_free[0]);  // dO rows 0..63: no later UMMA of this fill needs them
      } else {
        // key role of chunk 2t+1: queries of chunk 2t+1 (rows 64..127)
        mma_run(r1, mdesc(xs, 64), kRowStep, mdesc(zt, 64), kRowStep, id_kv, 4, true);
        ok = free_wait(hvv_free, n + 1);  // chunk 2t-1's dv columns read
        if (!ok) break;
        mma_run(r1 + 64, mdesc(do0, 64), kRowStep, mdesc(pt, 64), kRowStep, id_kv, 4, false);
        // dQ^T of chunk 2t+1 from the keys of chunk 2t+1
        mma_run(r1, mdesc(xs, 64), kRowStep, kdesc(zt + 64 * 128, 0), 32, id_q, 4, true);
        tc::umma_commit(pz_free);
        if (seg_end) tc::umma_commit(&hv_done[(n + 1) & 1]);
      }
      ++kb;
    }
    if (!ok) break;
    // (the dP UMMAs read dO too; each finished before the softmax loaded its block)
    if (!full) tc::umma_commit(do_free[0]);  // a half fill has one block
    else tc::umma_commit(do_free[1]);        // rows 64..: full fills only
    if (!full) tc::umma_commit(&slot_free[s]);  // the half fill's slot
    if (full) n += 2;
    ++F;
    f.advance(p);
  }
  uint64_t* done_bar = bars + Bars::kDone;
  tc::umma_commit(done_bar);
  att_tc::drain_wait(done_bar, 0);
}

template <int MASK>
__global__ void __launch_bounds__(kThreads, 1) attend_bwd_tc_kernel(const Params p) {
  constexpr bool CAUSAL = (MASK & kMaskCausal) != 0, BUCKET = (MASK & kMaskBucket) != 0;
  constexpr bool UNION = (MASK & kMaskUnion) != 0;
  using Lay = Layout;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte-aligned base as an offset from the shared array itself (stays a shared-memory pointer)
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* slot_full = bars + Bars::kSlotFull;
  uint64_t* slot_free = bars + Bars::kSlotFree;
  uint64_t* do_full[2] = {bars + Bars::kDoFull, bars + Bars::kDoFull1};
  uint64_t* do_free[2] = {bars + Bars::kDoFree, bars + Bars::kDoFree1};
  uint64_t* sp_full = bars + Bars::kSpFull;
  uint64_t* sp_free = bars + Bars::kSpFree;
  uint64_t* pz_full = bars + Bars::kPzFull;
  uint64_t* pz_free = bars + Bars::kPzFree;
  uint64_t* hv_done = bars + Bars::kHvDone;
  uint64_t* hvh_free = bars + Bars::kHvHFree;
  uint64_t* hvv_free = bars + Bars::kHvVFree;
  uint64_t* r_full = bars + Bars::kRFull;
  uint64_t* done_bar = bars + Bars::kDone;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);
  const float4* aux_s = reinterpret_cast<const float4*>(smem + Lay::kAux);
  const float* kinv_s = reinterpret_cast<const float*>(smem + Lay::kKinv);
  const int32_t* perm_s = reinterpret_cast<const int32_t*>(smem + Lay::kPerm);
  float* r_s = reinterpret_cast<float*>(smem + Lay::kR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&slot_full[i], 64);
      tc::mbar_init(&slot_free[i], 1);
      tc::mbar_init(&r_full[i], 256);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(do_full[i], 32);
      tc::mbar_init(do_free[i], 1);
    }
    tc::mbar_init(pz_full, 256);
    tc::mbar_init(pz_free, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sp_full[i], 1);
      tc::mbar_init(&sp_free[i], 256);
      tc::mbar_init(&hv_done[i], 1);
      tc::mbar_init(&hvh_free[2 * i], 128);
      tc::mbar_init(&hvh_free[2 * i + 1], 128);
      tc::mbar_init(&hvv_free[i], 128);
    }
    tc::mbar_init(done_bar, 2);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 2) tc::tmem_alloc(tmem_holder, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const long long L = p.L;

  if (warp < 4) {
    att_tc::setmaxnreg_dec<kLowRegs>();
    if (warp < 2) {
      // ------------------------------------------------------------ producers
      const int pw = warp;
      const uint32_t qk0 = tc::smem_u32(smem + Lay::kQK), v0 = tc::smem_u32(smem + Lay::kV);
      FillIt f;
      f.init(p);
      uint32_t F = 0, nd = 0;
      while (f.valid) {
        const int s = F & 1;
        int pos[2];
        const bool mine = fill_rows(p, f, pw, pos);
        if (!att_tc::warp_wait(&slot_free[s], ((F >> 1) & 1) ^ 1, abort_flag)) break;
        if (mine) {
          const long long rb = f.bh * L;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int i = 64 * pw + 32 * k + lane;
            const long long g = rb + pos[k];
            tc::cp_async16(tc::smem_u32(smem + Lay::kAux) + (s * kRows + i) * 16, p.aux + g);
            tc::cp_async4(tc::smem_u32(smem + Lay::kKinv) + (s * kRows + i) * 4,
                          reinterpret_cast<const float*>(p.aux + g) + 2);
            tc::cp_async4(tc::smem_u32(smem + Lay::kPerm) + (s * kRows + i) * 4,
                          p.perm + (f.bh * p.n_rounds + p.round) * L +
                              (f.kind == kLead ? 2 * f.t0 - 1 : 2 * f.t + (f.kind == kFull ? pw : 0)) * kC +
                              32 * k + lane);
            if (MASK != 0)  // the row's bucket in this round and whether its window leaves it alone
              tc::cp_async4(tc::smem_u32(smem + Lay::kMaskRow) + (s * kRows + i) * 4,
                            p.mask_rows + (f.bh * p.n_rounds + p.round) * L + pos[k]);
            if (MASK & kMaskUnion)  // every round's bucket of the row: one 16-byte packed row
              tc::cp_async16(tc::smem_u32(smem + Lay::kUnion) + (s * kRows + i) * 16, p.bk_rows + g);
          }
          gather64(qk0 + s * Lay::kTile, p.qk, rb, pw, pos);
          if (f.kind != kHalo) gather64(v0 + s * Lay::kTile, p.v, rb, pw, pos);
        }
        tc::cp_async_arrive(&slot_full[s]);
        // the fill's dO rows, once the UMMAs of the previous fill that read them are done: rows 0..63
        // for every fill with queries, rows 64.. for full fills (a half fill has none)
        if (f.kind != kLead && (pw == 0 || f.kind == kFull)) {
          if (!att_tc::warp_wait(do_free[pw], (nd & 1) ^ 1, abort_flag)) break;
          if (mine) gather64(tc::smem_u32(smem + Lay::kDO), p.dout, f.bh * L, pw, pos);
          tc::cp_async_arrive(do_full[pw]);
          ++nd;
        }
        ++F;
        f.advance(p);
      }
      asm volatile("cp.async.wait_all;" ::: "memory");  // never leave with copies in flight
    } else {
      // ------------------------------------------------------------ UMMA issuers
      if (lane == 0) {
        if (warp == 2)
          issuer_s(p, smem, tmem, abort_flag);
        else
          issuer_hv(p, smem, tmem, abort_flag);
      }
      __syncwarp();
    }
  } else if (warp < 12) {
    att_tc::setmaxnreg_inc<kSoftRegs>();
    // ------------------------------------------------------------ softmax
    const int wg = (warp - 4) >> 2;  // keys 32 wg .. 32 wg + 31 of each block
    const int q = warp & 3;
    const int i = 32 * q + lane;     // query row of the fill
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const float c2 = p.scale * 1.4426950408889634f;
    uint8_t* pz_p = smem + Lay::kP;
    uint8_t* pz_z = smem + Lay::kZ;
    FillIt f;
    f.init(p);
    uint32_t F = 0, kb = 0, ff = 0;
    bool ok = true;
    while (f.valid) {
      const uint32_t s = F & 1, sp = (F + 1) & 1;
      if (f.kind == kLead) {
        ++F;
        f.advance(p);
        continue;
      }
      const bool full = f.kind == kFull, has_prev = f.has_prev();
      ok = att_tc::warp_wait(&slot_full[s], (F >> 1) & 1, abort_flag) &&
           (!has_prev || att_tc::warp_wait(&slot_full[sp], ((F - 1) >> 1) & 1, abort_flag));
      if (!ok) break;
      // LSE log2 e and Delta of the row (a half fill has rows 0..63 only)
      const bool row_here = full || q < 2;
      const float4 qa = row_here ? aux_s[s * kRows + i] : make_float4(0.f, 0.f, 0.f, 0.f);
      // masks: the query's position, bucket, whether it is alone in its window, every round's bucket
      const int32_t* mrow = reinterpret_cast<const int32_t*>(smem + Lay::kMaskRow);
      const uint4* urow = reinterpret_cast<const uint4*>(smem + Lay::kUnion);
      const int qpos = (CAUSAL && row_here) ? perm_s[s * kRows + i] : 0;
      const int qm = (MASK != 0 && row_here) ? mrow[s * kRows + i] : 0;
      const bool alone = qm < 0;
      const int qb = qm & 0x7fffffff;
      __half2 qu[4];
      att_tc::union_query((UNION && row_here) ? urow[s * kRows + i] : make_uint4(0u, 0u, 0u, 0u), p.n_rounds, qu);
      float r = 0.f;                            // x_i . dQ_i over this warp group's keys
      int blocks[3], nb = 0;
      if (has_prev) blocks[nb++] = 0;
      if (full) {
        blocks[nb++] = 1;
        blocks[nb++] = 2;
      }
      for (int bi = 0; bi < nb; ++bi) {
        const int b = blocks[bi];
        const bool active = b == 1 || (b == 0 ? q < 2 : q >= 2);  // the block is in the row's window
        ok = att_tc::warp_wait(&sp_full[kb & 1], (kb >> 1) & 1, abort_flag);
        if (!ok) break;
        tc::tc_fence_after();
        uint32_t sr[32], dr[32];
        if (active) {
          const uint32_t spb = tmem + lane_base + (kb & 1) * kSPCols + 32 * wg;
          tc::tmem_ld32(spb, sr);
          tc::tmem_ld32(spb + kPOff, dr);
          tc::tmem_wait_ld_regs(sr);
          tc::tmem_wait_ld_regs(dr);
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&sp_free[kb & 1]);
        uint32_t pw16[16], zw16[16];
        if (active) {
          // keys of the block: slot and first row
          const int krow0 = (b == 0 ? sp * kRows + 64 : s * kRows + (b == 2 ? 64 : 0)) + 32 * wg;
          const float* kin = kinv_s + krow0;
          // own key: block 1 for rows 0..63, block 2 for rows 64..127, element `lane` of group wg == q % 2;
          // a row that its masks leave alone keeps it
          const bool self_grp = p.self_mask && !alone && b != 0 && (q & 1) == wg && (b == 1) == (q < 2);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 k4 = *reinterpret_cast<const float4*>(kin + e);
            const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
            float pe[4], ze[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float sv = __uint_as_float(sr[e + u]);
              float z2 = fmaf(sv, kv[u] * c2, -qa.x);
              if (UNION) z2 -= att_tc::union_log2(urow + krow0 + e + u, qu);  // log2 of the rounds shared
              float pv = tc::ex2_approx(z2);
              if (self_grp && e + u == lane) pv = 0.f;
              if (CAUSAL && perm_s[krow0 + e + u] > qpos) pv = 0.f;
              if (BUCKET && (mrow[krow0 + e + u] & 0x7fffffff) != qb) pv = 0.f;
              const float zv = pv * (__uint_as_float(dr[e + u]) - qa.y) * (kv[u] * p.scale);
              pe[u] = pv;
              ze[u] = zv;
            }
            pw16[e / 2] = tc::pack_bf16x2(pe[0], pe[1]);
            pw16[e / 2 + 1] = tc::pack_bf16x2(pe[2], pe[3]);
            zw16[e / 2] = tc::pack_bf16x2(ze[0], ze[1]);
            zw16[e / 2 + 1] = tc::pack_bf16x2(ze[2], ze[3]);
            // x_i . dQ_i with the rounded Z the UMMA sees
            const __nv_bfloat162 z01 = *reinterpret_cast<const __nv_bfloat162*>(&zw16[e / 2]);
            const __nv_bfloat162 z23 = *reinterpret_cast<const __nv_bfloat162*>(&zw16[e / 2 + 1]);
            r = fmaf(__low2float(z01), __uint_as_float(sr[e]), r);
            r = fmaf(__high2float(z01), __uint_as_float(sr[e + 1]), r);
            r = fmaf(__low2float(z23), __uint_as_float(sr[e + 2]), r);
            r = fmaf(__high2float(z23), __uint_as_float(sr[e + 3]), r);
          }
        }
        ok = att_tc::warp_wait(pz_free, (kb & 1) ^ 1, abort_flag);
        if (!ok) break;
        if (active) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t off = swz(i, 4 * wg + c);
            *reinterpret_cast<uint4*>(pz_p + off) =
                make_uint4(pw16[4 * c], pw16[4 * c + 1], pw16[4 * c + 2], pw16[4 * c + 3]);
            *reinterpret_cast<uint4*>(pz_z + off) =
                make_uint4(zw16[4 * c], zw16[4 * c + 1], zw16[4 * c + 2], zw16[4 * c + 3]);
          }
          tc::fence_proxy_async_smem();
        }
        tc::mbar_arrive(pz_full);
        ++kb;
      }
      if (!ok) break;
      if (full) {
        r_s[((ff & 1) * 2 + wg) * kRows + i] = r;
        tc::mbar_arrive(&r_full[ff & 1]);
        ++ff;
      }
      ++F;
      f.advance(p);
    }
  } else {
    att_tc::setmaxnreg_inc<kEpiRegs>();
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int d = 32 * q + lane;  // feature of this thread (TMEM lane)
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    float* xh = reinterpret_cast<float*>(smem + Lay::kXH);
    FillIt f;
    f.init(p);
    uint32_t n = 0, ff = 0;
    // every wait of the epilogue warps ends in one joint decision, so that their named barriers stay matched
    auto epi_wait = [&](uint64_t* bar, uint32_t parity) {
      return bar_and(1, 128, att_tc::warp_wait(bar, parity, abort_flag));
    };
    float* stage = reinterpret_cast<float*>(smem + Lay::kStage) + q * 32 * 32;  // this warp's [token][feature]
    // 32 tokens x this warp's 32 features from the staging tile to their rows (token t's position
    // in lane t of pos): 4 tokens per instruction, 16 bytes per lane; the first round stores,
    // later ones add in L2 (one writer per element and launch, launches in order: the sums do not
    // depend on timing)
    auto rows_out = [&](float* base, int pos) {
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int t = 4 * it + (lane >> 3), f4 = 4 * (lane & 7);
        const float4 val = *reinterpret_cast<const float4*>(stage + t * 32 + f4);
        float* dst = base + (long long)__shfl_sync(0xffffffffu, pos, t) * kD + f4;
        if (p.accumulate)
          red_add_v4(dst, val);
        else
          *reinterpret_cast<float4*>(dst) = val;
      }
    };
    // One finished chunk: TMEM region of owned chunk c, rows [row0, row0 + 64) of fill slot s, x . dQ
    // partials in r buffer rbuf.  What it needs from the slot is copied to registers first; a
    // chunk that is its slot's last reader (`last`) releases the slot before its arithmetic.
    auto chunk_out = [&](uint32_t c, uint32_t s, int row0, uint32_t rbuf, long long bh, bool last) -> bool {
      if (!epi_wait(&hv_done[c & 1], (c >> 1) & 1)) return false;
      tc::tc_fence_after();
      const uint16_t* xt = reinterpret_cast<const uint16_t*>(smem + Lay::kQK + s * Lay::kTile +
                                                             (d >> 6) * Lay::kHalf) + (d & 7);
      const int dc = (d & 63) >> 3;
      uint32_t xpk[32];  // bf16 x of tokens e (low half) and 32 + e (high half), feature d
#pragma unroll
      for (int e = 0; e < 32; ++e)
        xpk[e] = (uint32_t)xt[swz(row0 + e, dc) / 2] | ((uint32_t)xt[swz(row0 + 32 + e, dc) / 2] << 16);
      const int pos_a = perm_s[s * kRows + row0 + lane], pos_b = perm_s[s * kRows + row0 + 32 + lane];
      const float kc_a = aux_s[s * kRows + row0 + lane].w, kc_b = aux_s[s * kRows + row0 + 32 + lane].w;
      if (last) {
        tc::named_bar_sync(1, 128);
        if (threadIdx.x == 12 * 32) tc::mbar_arrive(&slot_free[s]);
      }
      const uint32_t reg = tmem + lane_base + kRegCol0 + (c & 1) * kRegCols;
      float* dq_w = p.dqk + bh * L * kD + 32 * q;  // this warp's 32 features
      float* dv_w = p.dv + bh * L * kD + 32 * q;
      // per 32-token half: its H columns (released once in registers: the next chunk of this region
      // writes them first), the key-normalisation term, the dqk rows; then the dv columns
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        auto xv = [&](int e) { return __uint_as_float(h ? (xpk[e] & 0xffff0000u) : (xpk[e] << 16)); };
        uint32_t hr[32];
        tc::tmem_ld32(reg + 32 * h, hr);
        tc::tmem_wait_ld_regs(hr);
        tc::tc_fence_before();
        tc::mbar_arrive(&hvh_free[(c & 1) * 2 + h]);
        float part;
        {
          float pr2[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) pr2[e] = xv(e) * __uint_as_float(hr[e]);
          part = transpose_reduce(pr2, lane);  // token 32 h + lane, this warp's 32 features
        }
        xh[q * 32 + lane] = part;
        tc::named_bar_sync(1, 128);
        const int row_l = row0 + 32 * h + lane;
        const float tot = xh[lane] + xh[32 + lane] + xh[64 + lane] + xh[96 + lane];
        const float rr = r_s[(rbuf * 2) * kRows + row_l] + r_s[(rbuf * 2 + 1) * kRows + row_l];
        const float coef = (tot - rr) * (h ? kc_b : kc_a);  // (x . G) (||x|| >= 1e-12) / ||x||^2
        tc::named_bar_sync(1, 128);  // xh is reused by the next half
#pragma unroll
        for (int e = 0; e < 32; ++e)
          stage[e * 32 + lane] = fmaf(-__shfl_sync(0xffffffffu, coef, e), xv(e), __uint_as_float(hr[e]));
        __syncwarp();
        rows_out(dq_w, h ? pos_b : pos_a);
        __syncwarp();
      }
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t vr[32];
        tc::tmem_ld32(reg + 64 + 32 * h, vr);
        tc::tmem_wait_ld_regs(vr);
        if (h == 1) {  // the region's last TMEM read
          tc::tc_fence_before();
          tc::mbar_arrive(&hvv_free[c & 1]);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) stage[e * 32 + lane] = __uint_as_float(vr[e]);
        __syncwarp();
        rows_out(dv_w, h ? pos_b : pos_a);
        __syncwarp();
      }
      return true;
    };
    uint32_t F = 0;
    while (f.valid) {
      const uint32_t s = F & 1, sp = (F + 1) & 1;
      if (f.kind == kLead) {
        ++F;
        f.advance(p);
        continue;
      }
      // chunk 2t-1 (rows 64.. of the previous slot, its last reader) finished by this fill's first block
      if (f.owns_prev() && !chunk_out(n - 1, sp, 64, (ff + 1) & 1, f.bh, true)) break;
      if (f.kind == kFull) {
        if (!epi_wait(&slot_full[s], (F >> 1) & 1) || !epi_wait(&r_full[ff & 1], (ff >> 1) & 1)) break;
        if (!chunk_out(n, s, 0, ff & 1, f.bh, false)) break;
        // segment end: chunk 2t+1 has no later queries
        if (f.t == p.n_fills - 1 && !chunk_out(n + 1, s, 64, ff & 1, f.bh, true)) break;
        n += 2;
        ++ff;
      }
      ++F;
      f.advance(p);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Masked backward, per (b, h, round) segment and sorted slot: the token's bucket in the round (for
// the bucket mask) and bit 31 set when its window (its own chunk of 64 and the previous one) holds
// no other key that the masks admit, so that the token keeps its own key (the self rule).  One CTA
// per pair of chunks with the chunk before it staged in shared memory; L % 128 == 0.
template <bool CAUSAL, bool BUCKET>
__global__ void __launch_bounds__(128) bwd_mask_rows_kernel(const int32_t* __restrict__ perm,
                                                            const int32_t* __restrict__ buckets, int L,
                                                            int32_t* __restrict__ mask_rows) {
  __shared__ int pos_s[192], bk_s[192];
  const int pairs = L / 128;
  const long long seg = blockIdx.x / pairs;
  const int base = (int)(blockIdx.x - seg * pairs) * 128;  // first slot of the pair
  const int32_t* pseg = perm + seg * L;
  for (int t = threadIdx.x; t < 192; t += 128) {
    const int slot = base - 64 + t;
    int pos = -1, bk = 0;
    if (slot >= 0) {
      pos = pseg[slot];
      if (BUCKET) bk = buckets[seg * L + pos];
    }
    pos_s[t] = pos;
    bk_s[t] = bk;
  }
  __syncthreads();
  const int me = 64 + threadIdx.x;              // this slot in the staged window
  const int w0 = threadIdx.x < 64 ? 0 : 64;     // its window: the previous chunk and its own
  const int mypos = pos_s[me], mybk = bk_s[me];
  bool other = false;
  for (int t = w0; t < w0 + 128 && !other; ++t)
    other = t != me && pos_s[t] >= 0 && (!CAUSAL || pos_s[t] < mypos) && (!BUCKET || bk_s[t] == mybk);
  mask_rows[seg * L + mypos] = (BUCKET ? mybk : 0) | (other ? 0 : (int)0x80000000u);
}

// Per-token terms of the backward: LSE log2 e, Delta = dout . out, 1/max(||x||, 1e-12)
// and the key-normalisation coefficient (||x|| >= 1e-12) / max(||x||, 1e-12)^2.
// One warp per token; D = 128, bf16 rows.
__global__ void bwd_aux_kernel(const __nv_bfloat16* __restrict__ qk, const __nv_bfloat16* __restrict__ out,
                               const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
                               float4* __restrict__ aux, long long n_tokens) {
  const long long tok = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (tok >= n_tokens) return;
  const int lane = threadIdx.x & 31;
  float x[4], o[4], g[4];
  load4_bf16(qk + tok * kD + 4 * lane, x);
  load4_bf16(out + tok * kD + 4 * lane, o);
  load4_bf16(dout + tok * kD + 4 * lane, g);
  float ss = 0.f, dl = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    ss = fmaf(x[e], x[e], ss);
    dl = fmaf(g[e], o[e], dl);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, off);
    dl += __shfl_xor_sync(0xffffffffu, dl, off);
  }
  if (lane == 0) {
    const float nrm = sqrtf(ss);
    const float kinv = 1.f / fmaxf(nrm, 1e-12f);
    aux[tok] = make_float4(lse[tok] * 1.4426950408889634f, dl, kinv, nrm >= 1e-12f ? kinv * kinv : 0.f);
  }
}

}  // namespace bwd_tc
}  // namespace lsh

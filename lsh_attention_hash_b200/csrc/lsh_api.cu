// C ABI entry points of the LSH attention library: argument validation and
// kernel dispatch.  Every compute step runs in the kernels included below.
#include <math.h>

#include <algorithm>
#include <mutex>
#include <stdint.h>

#include <cudaTypedefs.h>

#include "attend_bwd_simt.cuh"
#include "attend_bwd_tc.cuh"
#include "attend_simt.cuh"
#include "attend_tc.cuh"
#include "combine.cuh"
#include "common.cuh"
#include "hash_simt.cuh"
#include "hash_tc.cuh"
#include "lsh_attention_hash.h"
#include "sort.cuh"

namespace {


inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool valid_dtype(int d) { return d == LSH_F32 || d == LSH_BF16; }

inline size_t elt_size(int d) { return d == LSH_F32 ? 4 : 2; }

inline lsh_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}

// Common shape rules for row tensors [B, H, L, D].
inline lsh_status check_bhld(int B, int H, int L, int D) {
  if (B < 0 || H < 0 || L < 0) return LSH_ERR_SHAPE;
  if (D < 8 || D > 256 || (D % 8) != 0) return LSH_ERR_SHAPE;
  if (L > (1 << 24)) return LSH_ERR_SHAPE;
  return LSH_OK;
}

inline bool index_space_ok(int B, int H, int L, int n_rounds) {
  return (long long)B * H * n_rounds * L < (1ll << 31);
}

// Device properties of the current device, cached per device ordinal.
struct DevInfo {
  int major = 0, sms = 0;
};
inline DevInfo dev_info() {
  static DevInfo cache[64];
  static bool have[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DevInfo{};
  if (!have[dev]) {
    DevInfo d;
    cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = d;
    have[dev] = true;
  }
  return cache[dev];
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (the
// library does not link libcuda directly).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
inline EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    tried = true;
  }
  return fn;
}

// 2D bf16 view [rows, cols] with a box of box_cols x box_rows, 128-byte swizzle.
inline bool make_tile_map(CUtensorMap* map, const void* base, long long rows, long long cols, int box_cols,
                          int box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Whether the tensor-core hash serves this shape (see hash_tc.cuh): R[round]
// resident in shared memory (D * half * 2 <= 128 KB) or streamed in chunks of
// 256 columns (half a multiple of 256).
inline bool hash_tc_eligible(int dtype, int D, int half, int n_rounds, const DevInfo& di) {
  if (dtype != LSH_BF16 || di.major != 10 || (D != 64 && D != 128)) return false;
  if (half != 32 && (half % 64 != 0 || !(half <= 256 ? (half == 64 || half == 128 || half == 256) : half % 256 == 0)))
    return false;
  return n_rounds <= di.sms;
}
inline bool hash_tc_streams_r(int D, int half) { return (long long)D * half * 2 > 128 * 1024; }

template <int D, int NC, bool FLAG, int SPLIT, int RS, bool WIDE = false>
lsh_status launch_hash_tc(const void* qk, const void* R, int B, int H, int L, int n_rounds, int half,
                          int32_t* buckets, uint8_t* near_tie, cudaStream_t s, int sms) {
  using namespace lsh::hash_tc;
  const long long rows = (long long)B * H * L;
  CUtensorMap mx, mr;
  if (!make_tile_map(&mx, qk, rows, D, 64, kRows)) return LSH_ERR_CUDA;
  if (half >= 64) {
    if (!make_tile_map(&mr, R, (long long)n_rounds * D, half, 64, D)) return LSH_ERR_CUDA;
  } else {
    mr = mx;  // 32 columns: the kernel copies R[round] by plain loads and never reads this map
  }
  Params p;
  p.r = static_cast<const __nv_bfloat16*>(R);
  p.buckets = buckets;
  p.near_tie = near_tie;
  p.nrows = rows;
  p.L = L;
  p.n_rounds = n_rounds;
  p.half = half;
  p.nchunks = half / NC;
  p.n_tiles = (rows + kRows - 1) / kRows;
  p.per_round = (int)std::max<long long>(1, std::min<long long>(sms / n_rounds, p.n_tiles));
  p.key_mask = 0x7FFFFFF0u;
  const unsigned grid = (unsigned)(p.per_round * n_rounds);
  auto kfn = hash_tc_kernel<D, NC, FLAG, SPLIT, RS, WIDE>;
  const int smem = (int)Layout<D>::smem_bytes(half, NC, RS);
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return LSH_ERR_CUDA;
  kfn<<<grid, threads_for(SPLIT), smem, s>>>(mx, mr, p);
  return cudaGetLastError() == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}

template <int D>
lsh_status dispatch_hash_tc(const void* qk, const void* R, int B, int H, int L, int n_rounds, int half,
                            int32_t* buckets, uint8_t* near_tie, cudaStream_t s, int sms) {
#define LSH_HTC(NC, RS)                                                                                  \
  return near_tie                                                                                        \
             ? launch_hash_tc<D, NC, true, (NC >= 128 ? 4 : 2), RS>(qk, R, B, H, L, n_rounds, half, buckets, \
                                                                     near_tie, s, sms)                     \
             : launch_hash_tc<D, NC, false, (NC >= 128 ? 4 : 2), RS>(qk, R, B, H, L, n_rounds, half, buckets, \
                                                                      near_tie, s, sms)
  // streamed projection ring: 3 chunks of 32 KB at D 64, 2 of 64 KB at D 128; rounds of 4096 columns
  // or more without the near-tie flag take the group-maximum fast path
  if (hash_tc_streams_r(D, half) && !near_tie && half >= 4096)
    return launch_hash_tc<D, 256, false, 4, D == 64 ? 3 : 2, true>(qk, R, B, H, L, n_rounds, half, buckets, near_tie,
                                                                    s, sms);
  if (hash_tc_streams_r(D, half)) LSH_HTC(256, D == 64 ? 3 : 2);
  if (half == 32) {  // one epilogue part (32 columns)
    return near_tie ? launch_hash_tc<D, 32, true, 1, 0>(qk, R, B, H, L, n_rounds, half, buckets, near_tie, s, sms)
                    : launch_hash_tc<D, 32, false, 1, 0>(qk, R, B, H, L, n_rounds, half, buckets, near_tie, s, sms);
  }
  if (half == 64) LSH_HTC(64, 0);
  if (half == 128) LSH_HTC(128, 0);
  LSH_HTC(256, 0);
#undef LSH_HTC
}

// Tensor-core chunk attention (bf16, chunk 64, D 64 or 128) on sm_100.
template <int D, typename TO, int MASK>
lsh_status launch_attend_tc(const void* qk, const void* v, const void* qk_sorted, const void* v_sorted,
                            const int32_t* perm, const int32_t* buckets, int B, int H, int L, int n_rounds,
                            int self_mask, float scale, void* out, float* lse, cudaStream_t s, int sms) {
  constexpr bool kUnion = (MASK & lsh::att_tc::kMaskUnion) != 0;
  using namespace lsh::att_tc;
  const long long segs = (long long)B * H * n_rounds;
  const bool sorted = qk_sorted != nullptr;
  Params p;
  p.perm = perm;
  p.buckets = buckets;
  p.out = out;
  p.lse = lse;
  p.L = L;
  p.n_rounds = n_rounds;
  p.n_chunks = L / kC;
  p.n_steps = (p.n_chunks + 1) / 2;
  p.run = 32;
  p.units_per_seg = (p.n_steps + p.run - 1) / p.run;
  p.n_units = segs * p.units_per_seg;
  p.self_mask = self_mask;
  p.colscale = scale * 1.4426950408889634f;  // log2(e)
  p.sorted_input = sorted ? 1 : 0;
  p.qk = (const uint8_t*)(sorted ? qk_sorted : qk);
  p.v = (const uint8_t*)(sorted ? v_sorted : v);
  p.out_v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0 ? 1 : 0;
  p.bk_rows = nullptr;
  uint4* rows = nullptr;
  if (kUnion) {  // every round's bucket of each token in one 16-byte row (stream-ordered scratch)
    const long long n_tok = (long long)B * H * L;
    if (cudaMallocAsync(reinterpret_cast<void**>(&rows), (size_t)n_tok * sizeof(uint4), s) != cudaSuccess)
      return LSH_ERR_CUDA;
    union_rows_kernel<<<(unsigned)((n_tok + 255) / 256), 256, 0, s>>>(buckets, n_tok, n_rounds, L, rows);
    p.bk_rows = rows;
  }
  const unsigned grid = (unsigned)std::min<long long>(p.n_units, sms);
  auto kfn = attend_tc_kernel<D, TO, MASK>;
  const int smem = (int)Layout<D>::kSmem;
  lsh_status st = LSH_OK;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    st = LSH_ERR_CUDA;
  } else {
    kfn<<<grid, kThreads, smem, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) st = LSH_ERR_CUDA;
  }
  if (rows && cudaFreeAsync(rows, s) != cudaSuccess && st == LSH_OK) st = LSH_ERR_CUDA;
  return st;
}

// Tensor-core backward (bf16 rows and out / dout, D 128, chunk 64, L % 128 == 0; the union
// correction up to 8 rounds) on sm_100: per-token terms (and, with masks, per-slot mask rows and
// each token's buckets in every round) into stream-ordered scratch buffers, then one launch per round.
template <int MASK>
lsh_status launch_attend_bwd_tc(const void* qk, const void* v, const int32_t* perm, const int32_t* buckets, int B,
                                int H, int L, int n_rounds, int self_mask, float scale, const void* out,
                                const float* lse, const void* dout, float* dqk, float* dv, cudaStream_t s, int sms) {
  using namespace lsh::bwd_tc;
  constexpr bool kCausal = (MASK & kMaskCausal) != 0, kBucket = (MASK & kMaskBucket) != 0;
  constexpr bool kUnion = (MASK & kMaskUnion) != 0;
  auto kfn = attend_bwd_tc_kernel<MASK>;
  // the setmaxnreg split hands out exactly the registers the launch holds: 512 threads x 128
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kfn) != cudaSuccess || fa.numRegs != 128) return LSH_ERR_UNSUPPORTED;
  const long long bhs = (long long)B * H, n_tok = bhs * L;
  float4* aux = nullptr;
  int32_t* mask_rows = nullptr;
  uint4* bk_rows = nullptr;
  lsh_status st = LSH_OK;
  if (cudaMallocAsync(reinterpret_cast<void**>(&aux), (size_t)n_tok * sizeof(float4), s) != cudaSuccess ||
      (MASK != 0 && cudaMallocAsync(reinterpret_cast<void**>(&mask_rows), (size_t)n_tok * n_rounds * 4, s) !=
                        cudaSuccess) ||
      (kUnion && cudaMallocAsync(reinterpret_cast<void**>(&bk_rows), (size_t)n_tok * sizeof(uint4), s) != cudaSuccess))
    st = LSH_ERR_CUDA;
  if (st == LSH_OK) {
    const int warps = 8;
    bwd_aux_kernel<<<(unsigned)((n_tok + warps - 1) / warps), warps * 32, 0, s>>>(
        (const __nv_bfloat16*)qk, (const __nv_bfloat16*)out, (const __nv_bfloat16*)dout, lse, aux, n_tok);
    if (MASK != 0)
      bwd_mask_rows_kernel<kCausal, kBucket><<<(unsigned)((L / 128) * bhs * n_rounds), 128, 0, s>>>(perm, buckets, L,
                                                                                                  mask_rows);
    if (kUnion)
      lsh::att_tc::union_rows_kernel<<<(unsigned)((n_tok + 255) / 256), 256, 0, s>>>(buckets, n_tok, n_rounds, L,
                                                                                    bk_rows);
    Params p;
    p.qk = (const uint8_t*)qk;
    p.v = (const uint8_t*)v;
    p.dout = (const uint8_t*)dout;
    p.perm = perm;
    p.aux = aux;
    p.dqk = dqk;
    p.dv = dv;
    p.L = L;
    p.n_rounds = n_rounds;
    p.n_fills = L / kRows;
    p.run = 16;
    p.units_per_seg = (p.n_fills + p.run - 1) / p.run;
    p.n_units = bhs * p.units_per_seg;
    p.self_mask = self_mask;
    p.scale = scale;
    p.mask_rows = mask_rows;
    p.bk_rows = bk_rows;
    const unsigned grid = (unsigned)std::min<long long>(p.n_units, sms);
    const int smem = (int)Layout::smem(kUnion);
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      st = LSH_ERR_CUDA;
    for (int r = 0; st == LSH_OK && r < n_rounds; ++r) {  // rounds in order: each token has one writer per launch
      p.round = r;
      p.accumulate = r > 0 ? 1 : 0;
      kfn<<<grid, kThreads, smem, s>>>(p);
      if (cudaGetLastError() != cudaSuccess) st = LSH_ERR_CUDA;
    }
  }
  for (void* ptr : {static_cast<void*>(aux), static_cast<void*>(mask_rows), static_cast<void*>(bk_rows)})
    if (ptr && cudaFreeAsync(ptr, s) != cudaSuccess && st == LSH_OK) st = LSH_ERR_CUDA;
  return st;
}

}  // namespace

extern "C" {

int lsh_abi_version(void) { return 2; }

const char* lsh_status_string(int s) {
  switch (s) {
    case LSH_OK: return "LSH_OK";
    case LSH_ERR_INVALID_ARG: return "LSH_ERR_INVALID_ARG";
    case LSH_ERR_SHAPE: return "LSH_ERR_SHAPE";
    case LSH_ERR_DTYPE: return "LSH_ERR_DTYPE";
    case LSH_ERR_ALIGN: return "LSH_ERR_ALIGN";
    case LSH_ERR_WORKSPACE: return "LSH_ERR_WORKSPACE";
    case LSH_ERR_CUDA: return "LSH_ERR_CUDA";
    case LSH_ERR_TIMEOUT: return "LSH_ERR_TIMEOUT";
    case LSH_ERR_UNSUPPORTED: return "LSH_ERR_UNSUPPORTED";
    default: return "LSH_ERR_UNKNOWN";
  }
}

lsh_status lsh_hash(const void* qk, int dtype, int B, int H, int L, int D, const void* R,
                    int n_rounds, int n_buckets, int32_t* buckets, uint8_t* near_tie, void* stream) {
  if (!valid_dtype(dtype)) return LSH_ERR_DTYPE;
  lsh_status st = check_bhld(B, H, L, D);
  if (st != LSH_OK) return st;
  if (n_rounds < 1 || n_buckets < 2 || n_buckets > 65536 || (n_buckets & 1)) return LSH_ERR_SHAPE;
  if (!index_space_ok(B, H, L, n_rounds)) return LSH_ERR_SHAPE;
  if (!qk || !R || !buckets) return LSH_ERR_INVALID_ARG;
  if (!aligned16(qk) || !aligned16(R) || !aligned16(buckets) || (near_tie && !aligned16(near_tie)))
    return LSH_ERR_ALIGN;
  const long long nrows = (long long)B * H * L;
  if (nrows == 0) return LSH_OK;
  const int half = n_buckets / 2;
  const DevInfo di = dev_info();
  if (hash_tc_eligible(dtype, D, half, n_rounds, di)) {
    cudaStream_t s = as_stream(stream);
    if (D == 128) return dispatch_hash_tc<128>(qk, R, B, H, L, n_rounds, half, buckets, near_tie, s, di.sms);
    return dispatch_hash_tc<64>(qk, R, B, H, L, n_rounds, half, buckets, near_tie, s, di.sms);
  }
  dim3 grid((unsigned)((nrows + lsh::kHashRows - 1) / lsh::kHashRows), (unsigned)n_rounds);
  const size_t smem = (size_t)lsh::kHashRows * D * sizeof(float);
  cudaStream_t s = as_stream(stream);
  if (dtype == LSH_F32)
    lsh::hash_simt_kernel<float><<<grid, lsh::kHashThreads, smem, s>>>(
        (const float*)qk, (const float*)R, nrows, L, D, n_rounds, half, buckets, near_tie);
  else
    lsh::hash_simt_kernel<__nv_bfloat16><<<grid, lsh::kHashThreads, smem, s>>>(
        (const __nv_bfloat16*)qk, (const __nv_bfloat16*)R, nrows, L, D, n_rounds, half, buckets,
        near_tie);
  return launch_status();
}

// Radix sort of segs segments of L positions (longer than one CTA sorts, or with more buckets), in
// the workspace ws (lsh::radix_ws words).
static lsh_status launch_radix_sort(const int32_t* buckets, long long segs, int L, int n_buckets, int32_t* perm,
                                    int32_t* inv, uint32_t* ws, cudaStream_t s) {
  const lsh::RadixWs w = lsh::radix_ws(segs, L, n_buckets);
  const int nt = lsh::radix_tiles(L);
  const long long n = (long long)lsh::kRadixDigits * nt;
  const int nch = lsh::sort_scan_chunks(segs, n);
  const long long C = (n + nch - 1) / nch;
  uint32_t* cnt = ws + w.cnt;
  uint32_t* sums = ws + w.sums;
  uint32_t* valid = ws + w.valid;
  int32_t* keys1 = reinterpret_cast<int32_t*>(ws + w.keys);
  int32_t* pos1 = reinterpret_cast<int32_t*>(ws + w.pos);
  const dim3 grid((unsigned)segs, nt), scan_grid((unsigned)segs, nch);
  const int threads = lsh::kRadixWarps * 32;
  const bool two = lsh::radix_passes(n_buckets) > 1;
  // pass 1: the low digit of the bucket ids
  lsh::radix_count_kernel<true><<<grid, threads, 0, s>>>(buckets, L, n_buckets, 0, nullptr, cnt);
  lsh::sort_chunk_sum_kernel<<<scan_grid, 1024, 0, s>>>(cnt, n, C, sums);
  lsh::sort_scan_kernel<<<scan_grid, 1024, 0, s>>>(cnt, n, C, sums, valid);
  if (two)
    lsh::radix_scatter_kernel<true, false><<<grid, threads, 0, s>>>(buckets, nullptr, L, n_buckets, 0, nullptr, cnt,
                                                                    keys1, pos1, nullptr);
  else
    lsh::radix_scatter_kernel<true, true><<<grid, threads, 0, s>>>(buckets, nullptr, L, n_buckets, 0, nullptr, cnt,
                                                                   nullptr, perm, inv);
  if (cudaGetLastError() != cudaSuccess) return LSH_ERR_CUDA;
  if (!two) return LSH_OK;
  // pass 2: the high digit, over the valid ids in the first pass's order
  const int shift = lsh::kRadixBits;
  lsh::radix_count_kernel<false><<<grid, threads, 0, s>>>(keys1, L, n_buckets, shift, valid, cnt);
  lsh::sort_chunk_sum_kernel<<<scan_grid, 1024, 0, s>>>(cnt, n, C, sums);
  lsh::sort_scan_kernel<<<scan_grid, 1024, 0, s>>>(cnt, n, C, sums, nullptr);
  lsh::radix_scatter_kernel<false, true><<<grid, threads, 0, s>>>(keys1, pos1, L, n_buckets, shift, valid, cnt,
                                                                  nullptr, perm, inv);
  return cudaGetLastError() == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}

// Shapes sorted by one CTA per segment (no workspace).
static inline bool sort_by_segment(int L, int n_buckets) {
  return L <= lsh::kSegMaxL && n_buckets <= lsh::kSegMaxBuckets;
}

size_t lsh_sort_workspace_bytes(int B, int H, int L, int n_rounds, int n_buckets) {
  if (B <= 0 || H <= 0 || L <= 0 || n_rounds <= 0 || n_buckets < 2) return 0;
  if (sort_by_segment(L, n_buckets)) return 0;
  return (size_t)lsh::radix_ws((long long)B * H * n_rounds, L, n_buckets).words * sizeof(uint32_t);
}

lsh_status lsh_sort_permute(const int32_t* buckets, int B, int H, int L, int n_rounds,
                            int n_buckets, int32_t* perm, int32_t* inv, const void* qk,
                            const void* v, int dtype, int D, void* qk_sorted, void* v_sorted,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 0 || H < 0 || L < 0 || L > (1 << 24)) return LSH_ERR_SHAPE;
  if (n_rounds < 1 || n_buckets < 2 || n_buckets > 65536 || (n_buckets & 1)) return LSH_ERR_SHAPE;
  if (!index_space_ok(B, H, L, n_rounds)) return LSH_ERR_SHAPE;
  if (!buckets || !perm) return LSH_ERR_INVALID_ARG;
  const bool gather = qk || v || qk_sorted || v_sorted;
  if (gather) {
    if (!qk || !v || !qk_sorted || !v_sorted) return LSH_ERR_INVALID_ARG;
    if (!valid_dtype(dtype)) return LSH_ERR_DTYPE;
    lsh_status st = check_bhld(B, H, L, D);
    if (st != LSH_OK) return st;
    if (!aligned16(qk) || !aligned16(v) || !aligned16(qk_sorted) || !aligned16(v_sorted))
      return LSH_ERR_ALIGN;
  }
  if (!aligned16(buckets) || !aligned16(perm) || (inv && !aligned16(inv))) return LSH_ERR_ALIGN;
  const long long segs = (long long)B * H * n_rounds;
  if (segs == 0 || L == 0) return LSH_OK;
  const size_t need = lsh_sort_workspace_bytes(B, H, L, n_rounds, n_buckets);
  if (need > 0 && (!workspace || workspace_bytes < need)) return LSH_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return LSH_ERR_ALIGN;

  cudaStream_t s = as_stream(stream);
  if (sort_by_segment(L, n_buckets)) {
    const size_t smem = lsh::sort_segment_smem(L, n_buckets);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(lsh::sort_segment_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
      return LSH_ERR_CUDA;
    lsh::sort_segment_kernel<<<(unsigned)segs, lsh::kSegWarps * 32, smem, s>>>(buckets, L, n_buckets, perm, inv);
    if (cudaGetLastError() != cudaSuccess) return LSH_ERR_CUDA;
  } else {
    const lsh_status st = launch_radix_sort(buckets, segs, L, n_buckets, perm, inv, (uint32_t*)workspace, s);
    if (st != LSH_OK) return st;
  }
  if (gather) {
    const int row_bytes = D * (int)elt_size(dtype);
    const long long nrows = segs * L;
    const long long work = nrows * (row_bytes / 16);
    const unsigned blocks = (unsigned)min((work + 255) / 256, 148ll * 64);
    lsh::gather_rows_kernel<<<blocks, 256, 0, s>>>((const uint8_t*)qk, perm, nrows, L, n_rounds,
                                                   row_bytes, (uint8_t*)qk_sorted);
    lsh::gather_rows_kernel<<<blocks, 256, 0, s>>>((const uint8_t*)v, perm, nrows, L, n_rounds,
                                                   row_bytes, (uint8_t*)v_sorted);
  }
  return launch_status();
}

}  // extern "C"

namespace {

// Scratch of lsh_sort_permute_noalloc: static device memory of this library,
// 16 MiB of 32-bit words (the radix sort's counters and, with two passes, the
// first pass's ids and positions) on every device that loads it.
constexpr size_t kNoallocScratchWords = (size_t)4 << 20;
__device__ __align__(256) uint32_t g_noalloc_scratch[kNoallocScratchWords];

// Device address of g_noalloc_scratch, looked up once per device with that
// device current (in host code the array's name is only a host-side stand-in).
uint32_t* noalloc_scratch_ptr() {
  static std::mutex mu;
  static uint32_t* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<uint32_t*>(p);
  }
  return ptrs[dev];
}

}  // namespace

extern "C" {

lsh_status lsh_sort_permute_noalloc(const int32_t* buckets, int B, int H, int L, int n_rounds,
                                    int n_buckets, int32_t* perm, int32_t* inv, void* stream) {
  if (B < 0 || H < 0 || L < 0 || L > (1 << 24)) return LSH_ERR_SHAPE;
  if (n_rounds < 1 || n_buckets < 2 || n_buckets > 65536 || (n_buckets & 1)) return LSH_ERR_SHAPE;
  if (!index_space_ok(B, H, L, n_rounds)) return LSH_ERR_SHAPE;
  if (!buckets || !perm) return LSH_ERR_INVALID_ARG;
  if (!aligned16(buckets) || !aligned16(perm) || (inv && !aligned16(inv))) return LSH_ERR_ALIGN;
  const long long segs = (long long)B * H * n_rounds;
  if (segs == 0 || L == 0) return LSH_OK;
  cudaStream_t s = as_stream(stream);
  if (sort_by_segment(L, n_buckets)) {
    // one CTA per segment, all state in shared memory: no scratch at all
    const size_t smem = lsh::sort_segment_smem(L, n_buckets);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(lsh::sort_segment_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
      return LSH_ERR_CUDA;
    lsh::sort_segment_kernel<<<(unsigned)segs, lsh::kSegWarps * 32, smem, s>>>(buckets, L, n_buckets, perm, inv);
    return launch_status();
  }
  const size_t words = (size_t)lsh::radix_ws(segs, L, n_buckets).words;
  if (words > kNoallocScratchWords) return LSH_ERR_WORKSPACE;
  uint32_t* ws = noalloc_scratch_ptr();
  if (!ws) return LSH_ERR_CUDA;
  const lsh_status st = launch_radix_sort(buckets, segs, L, n_buckets, perm, inv, ws, s);
  if (st != LSH_OK) return st;
  return launch_status();
}

lsh_status lsh_chunk_attend(const void* qk, const void* v, int dtype, int B, int H, int L, int D,
                            int n_rounds, const int32_t* perm, const int32_t* buckets,
                            const void* qk_sorted, const void* v_sorted, int chunk, int mask, float scale,
                            void* out_rounds, int out_dtype, float* lse, void* stream) {
  if (!valid_dtype(dtype) || !valid_dtype(out_dtype)) return LSH_ERR_DTYPE;
  lsh_status st = check_bhld(B, H, L, D);
  if (st != LSH_OK) return st;
  if (n_rounds < 1 || !index_space_ok(B, H, L, n_rounds)) return LSH_ERR_SHAPE;
  if (chunk < 1 || (L > 0 && (chunk > L || L % chunk != 0))) return LSH_ERR_SHAPE;
  if (mask < 0 || mask > (LSH_MASK_SELF | LSH_MASK_CAUSAL | LSH_MASK_BUCKET | LSH_MASK_UNION))
    return LSH_ERR_INVALID_ARG;
  const int self_mask = (mask & LSH_MASK_SELF) ? 1 : 0;
  const int causal = (mask & LSH_MASK_CAUSAL) ? 1 : 0;
  const int bucket_mask = (mask & LSH_MASK_BUCKET) ? 1 : 0;
  const int union_count = (mask & LSH_MASK_UNION) ? 1 : 0;
  if (union_count && !bucket_mask) return LSH_ERR_INVALID_ARG;
  if (bucket_mask && !buckets) return LSH_ERR_INVALID_ARG;
  if (buckets && !aligned16(buckets)) return LSH_ERR_ALIGN;
  if (!qk || !v || !perm || !out_rounds || !lse) return LSH_ERR_INVALID_ARG;
  if ((qk_sorted == nullptr) != (v_sorted == nullptr)) return LSH_ERR_INVALID_ARG;
  if (!aligned16(qk) || !aligned16(v) || !aligned16(perm) || !aligned16(out_rounds) ||
      !aligned16(lse) || (qk_sorted && (!aligned16(qk_sorted) || !aligned16(v_sorted))))
    return LSH_ERR_ALIGN;
  const long long segs = (long long)B * H * n_rounds;
  if (segs == 0 || L == 0) return LSH_OK;
  if (segs > 65535) return LSH_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)D);
  cudaStream_t s = as_stream(stream);

  const DevInfo di = dev_info();
  if (dtype == LSH_BF16 && chunk == lsh::att_tc::kC && (D == 64 || D == 128) && di.major == 10 &&
      (!union_count || n_rounds <= lsh::att_tc::kUnionRounds)) {
    using lsh::att_tc::kMaskBucket;
    using lsh::att_tc::kMaskCausal;
    using lsh::att_tc::kMaskUnion;
#define LSH_ATT_TC_M(DD, TO, MM)                                                                            \
  return launch_attend_tc<DD, TO, MM>(qk, v, qk_sorted, v_sorted, perm, buckets, B, H, L, n_rounds, self_mask, \
                                      scale, out_rounds, lse, s, di.sms)
#define LSH_ATT_TC(DD, TO)                                                              \
  do {                                                                                  \
    if (union_count && causal) LSH_ATT_TC_M(DD, TO, kMaskCausal | kMaskBucket | kMaskUnion); \
    if (union_count) LSH_ATT_TC_M(DD, TO, kMaskBucket | kMaskUnion);                    \
    if (causal && bucket_mask) LSH_ATT_TC_M(DD, TO, kMaskCausal | kMaskBucket);         \
    if (causal) LSH_ATT_TC_M(DD, TO, kMaskCausal);                                      \
    if (bucket_mask) LSH_ATT_TC_M(DD, TO, kMaskBucket);                                 \
    LSH_ATT_TC_M(DD, TO, 0);                                                            \
  } while (0)
    if (D == 128) {
      if (out_dtype == LSH_BF16) LSH_ATT_TC(128, __nv_bfloat16); else LSH_ATT_TC(128, float);
    } else {
      if (out_dtype == LSH_BF16) LSH_ATT_TC(64, __nv_bfloat16); else LSH_ATT_TC(64, float);
    }
#undef LSH_ATT_TC
#undef LSH_ATT_TC_M
  }

  const int qb_per_chunk = (chunk + lsh::kAttQ - 1) / lsh::kAttQ;
  dim3 grid((unsigned)((L / chunk) * qb_per_chunk), (unsigned)segs);
  const size_t smem = ((size_t)lsh::kAttQ * (D + 1) + lsh::kAttK * (D + 1) + lsh::kAttK * D + lsh::kAttK +
                        (union_count ? (size_t)n_rounds * (lsh::kAttK + lsh::kAttQ) : 0)) * 4;
  if (smem > (size_t)227 * 1024) return LSH_ERR_UNSUPPORTED;  // union with very many rounds
  const int threads = lsh::kAttWarps * 32;
#define LSH_ATT(T, TO)                                                                          \
  do {                                                                                           \
    auto kfn = lsh::attend_simt_kernel<T, TO>;                                                   \
    if (smem > 48 * 1024) cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    kfn<<<grid, threads, smem, s>>>((const T*)qk, (const T*)v, perm, buckets, (const T*)qk_sorted, \
                                    (const T*)v_sorted, L, D, n_rounds, chunk, self_mask, causal,  \
                                    bucket_mask, union_count, scale, (TO*)out_rounds, lse);      \
  } while (0)
  if (dtype == LSH_F32) {
    if (out_dtype == LSH_F32) LSH_ATT(float, float); else LSH_ATT(float, __nv_bfloat16);
  } else {
    if (out_dtype == LSH_F32) LSH_ATT(__nv_bfloat16, float); else LSH_ATT(__nv_bfloat16, __nv_bfloat16);
  }
#undef LSH_ATT
  return launch_status();
}

lsh_status lsh_chunk_attend_backward(const void* qk, const void* v, int dtype, int B, int H, int L, int D,
                                     int n_rounds, const int32_t* perm, const int32_t* buckets, int chunk,
                                     int mask, float scale, const void* out, const float* lse,
                                     const void* dout, int out_dtype, float* dqk, float* dv, void* stream) {
  if (!valid_dtype(dtype) || !valid_dtype(out_dtype)) return LSH_ERR_DTYPE;
  lsh_status st = check_bhld(B, H, L, D);
  if (st != LSH_OK) return st;
  if (n_rounds < 1 || !index_space_ok(B, H, L, n_rounds)) return LSH_ERR_SHAPE;
  if (chunk < 1 || (L > 0 && (chunk > L || L % chunk != 0))) return LSH_ERR_SHAPE;
  if (mask < 0 || mask > (LSH_MASK_SELF | LSH_MASK_CAUSAL | LSH_MASK_BUCKET | LSH_MASK_UNION))
    return LSH_ERR_INVALID_ARG;
  const int self_mask = (mask & LSH_MASK_SELF) ? 1 : 0;
  const int causal = (mask & LSH_MASK_CAUSAL) ? 1 : 0;
  const int bucket_mask = (mask & LSH_MASK_BUCKET) ? 1 : 0;
  const int union_count = (mask & LSH_MASK_UNION) ? 1 : 0;
  if (union_count && !bucket_mask) return LSH_ERR_INVALID_ARG;
  if (bucket_mask && !buckets) return LSH_ERR_INVALID_ARG;
  if (!qk || !v || !perm || !out || !lse || !dout || !dqk || !dv) return LSH_ERR_INVALID_ARG;
  if (!aligned16(qk) || !aligned16(v) || !aligned16(perm) || !aligned16(out) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dqk) || !aligned16(dv) || (buckets && !aligned16(buckets)))
    return LSH_ERR_ALIGN;
  const long long bhs = (long long)B * H;
  if (bhs == 0 || L == 0) return LSH_OK;
  if (bhs > 65535) return LSH_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)D);
  const size_t smem = lsh::bwd_smem_words(D, n_rounds, union_count) * 4;
  if (smem > (size_t)227 * 1024) return LSH_ERR_UNSUPPORTED;  // union with very many rounds
  cudaStream_t s = as_stream(stream);
  const DevInfo di = dev_info();
  if (di.major == 10 && dtype == LSH_BF16 && out_dtype == LSH_BF16 && D == 128 && chunk == 64 && L % 128 == 0 &&
      (!union_count || n_rounds <= lsh::att_tc::kUnionRounds)) {
    using lsh::bwd_tc::kMaskBucket;
    using lsh::bwd_tc::kMaskCausal;
    using lsh::bwd_tc::kMaskUnion;
#define LSH_BWD_TC(MM)                                                                                         \
  return launch_attend_bwd_tc<MM>(qk, v, perm, buckets, B, H, L, n_rounds, self_mask, scale, out, lse, dout, dqk, \
                                  dv, s, di.sms)
    if (union_count && causal) LSH_BWD_TC(kMaskCausal | kMaskBucket | kMaskUnion);
    if (union_count) LSH_BWD_TC(kMaskBucket | kMaskUnion);
    if (causal && bucket_mask) LSH_BWD_TC(kMaskCausal | kMaskBucket);
    if (causal) LSH_BWD_TC(kMaskCausal);
    if (bucket_mask) LSH_BWD_TC(kMaskBucket);
    LSH_BWD_TC(0);
#undef LSH_BWD_TC
  }
  const size_t grad_bytes = (size_t)bhs * L * D * sizeof(float);
  if (cudaMemsetAsync(dqk, 0, grad_bytes, s) != cudaSuccess || cudaMemsetAsync(dv, 0, grad_bytes, s) != cudaSuccess)
    return LSH_ERR_CUDA;
  const int blocks_per_chunk = (chunk + lsh::kBwdB - 1) / lsh::kBwdB;
  dim3 grid((unsigned)((L / chunk) * blocks_per_chunk), (unsigned)bhs);
  const int threads = lsh::kBwdWarps * 32;
#define LSH_BWD(T, TO)                                                                                   \
  do {                                                                                                    \
    auto kfn = D <= 128 ? lsh::attend_bwd_simt_kernel<T, TO, 4> : lsh::attend_bwd_simt_kernel<T, TO, 8>;  \
    if (smem > 48 * 1024 &&                                                                               \
        cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)  \
      return LSH_ERR_CUDA;                                                                                \
    for (int r = 0; r < n_rounds; ++r) /* rounds in order: every token has one writer per launch */      \
      kfn<<<grid, threads, smem, s>>>((const T*)qk, (const T*)v, perm, buckets, (const TO*)out, lse,      \
                                      (const TO*)dout, L, D, n_rounds, r, chunk, self_mask, causal,       \
                                      bucket_mask, union_count, scale, dqk, dv);                          \
  } while (0)
  if (dtype == LSH_F32) {
    if (out_dtype == LSH_F32) LSH_BWD(float, float); else LSH_BWD(float, __nv_bfloat16);
  } else {
    if (out_dtype == LSH_F32) LSH_BWD(__nv_bfloat16, float); else LSH_BWD(__nv_bfloat16, __nv_bfloat16);
  }
#undef LSH_BWD
  return launch_status();
}

lsh_status lsh_combine_rounds(const void* out_rounds, int in_dtype, const float* lse, int B, int H,
                              int L, int D, int n_rounds, void* out, int out_dtype, float* lse_out,
                              void* stream) {
  if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return LSH_ERR_DTYPE;
  lsh_status st = check_bhld(B, H, L, D);
  if (st != LSH_OK) return st;
  if (n_rounds < 1 || !index_space_ok(B, H, L, n_rounds)) return LSH_ERR_SHAPE;
  if (!out_rounds || !lse || !out) return LSH_ERR_INVALID_ARG;
  if (!aligned16(out_rounds) || !aligned16(lse) || !aligned16(out) || (lse_out && !aligned16(lse_out)))
    return LSH_ERR_ALIGN;
  const long long ntok = (long long)B * H * L;
  if (ntok == 0) return LSH_OK;
  const long long threads_total = ntok * (D / 8);
  const unsigned blocks = (unsigned)((threads_total + 255) / 256);
  cudaStream_t s = as_stream(stream);
  const int G = D / 8;
  const bool g_pow2 = (G & (G - 1)) == 0;
  const int NR = (g_pow2 && n_rounds <= G && (n_rounds == 1 || n_rounds == 2 || n_rounds == 4 || n_rounds == 8))
                     ? n_rounds : 0;
#define LSH_CMB_NR(TI, TO, NRV)                                                                       \
  lsh::combine_kernel<TI, TO, NRV><<<blocks, 256, 0, s>>>((const TI*)out_rounds, lse, ntok, L, D, n_rounds, \
                                                          (TO*)out, lse_out)
#define LSH_CMB(TI, TO)                   \
  do {                                    \
    switch (NR) {                         \
      case 1: LSH_CMB_NR(TI, TO, 1); break; \
      case 2: LSH_CMB_NR(TI, TO, 2); break; \
      case 4: LSH_CMB_NR(TI, TO, 4); break; \
      case 8: LSH_CMB_NR(TI, TO, 8); break; \
      default: LSH_CMB_NR(TI, TO, 0); break; \
    }                                     \
  } while (0)
  if (in_dtype == LSH_F32) {
    if (out_dtype == LSH_F32) LSH_CMB(float, float); else LSH_CMB(float, __nv_bfloat16);
  } else {
    if (out_dtype == LSH_F32) LSH_CMB(__nv_bfloat16, float); else LSH_CMB(__nv_bfloat16, __nv_bfloat16);
  }
#undef LSH_CMB_NR
#undef LSH_CMB
  return launch_status();
}

lsh_status lsh_get_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return LSH_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, lsh::g_status, sizeof(int)) != cudaSuccess) return LSH_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(lsh::g_status, &zero, sizeof(int)) != cudaSuccess) return LSH_ERR_CUDA;
  }
  return (lsh_status)h;
}

}  // extern "C"

/*
 * lsh_attention_hash.h -- C ABI of the B200 (sm_100a) shared-QK LSH attention
 * forward pass (the Reformer's LSH attention).
 *
 * The method, as the pages state it:
 *   - Ultralytics glossary "Reformer", section "Atencao LSH": one shared
 *     projection for queries and keys; each vector is hashed by multiplying
 *     with a random matrix R and taking as bucket the position of the largest
 *     value of [xR, -xR]; tokens are sorted by bucket, the sorted sequence is
 *     cut into equal blocks and each token attends to its own block and the
 *     previous one; several hash rounds run in parallel.
 *   - twgreatdaily ICLR 2020 Reformer article, section "1 LSH Attention":
 *     attention of a query as a sum over its admissible key set divided by the
 *     set's partition function; Q = K with length-normalised keys; two-level
 *     sort by (bucket, position); a later chunk looks back one chunk; several
 *     rounds with different hash functions.
 *   - ai-scholar.tech Reformer article, "Transformerの問題点とは": the
 *     1/sqrt(d_k) logit scale.
 *
 * Conventions shared by every call:
 *   - Tensors are dense, row-major, caller-owned device buffers; every pointer
 *     must be 16-byte aligned.  The library never allocates or frees device
 *     memory: scratch space is passed in by the caller (size from the matching
 *     *_workspace_bytes query).
 *   - Shapes: B batch, H heads, L sequence length, D head dim, n_rounds hash
 *     rounds.  Index tensors are int32, so B*H*n_rounds*L < 2^31.
 *   - dtype codes: LSH_F32 (float) or LSH_BF16 (bfloat16); accumulation is
 *     always fp32.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and does no host synchronisation, except
 *     lsh_get_device_status.
 *   - Argument, shape, dtype and alignment errors are returned before any
 *     launch and leave every output untouched.  A failed launch returns
 *     LSH_ERR_CUDA.  Errors that kernels detect (an exhausted bounded wait)
 *     are recorded in a per-device status word read by lsh_get_device_status.
 *   - An empty problem (B*H*L == 0) returns LSH_OK without launching.
 *   - No C++ exception crosses this boundary.
 */
#ifndef LSH_ATTENTION_HASH_H
#define LSH_ATTENTION_HASH_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LSH_API __attribute__((visibility("default")))
#else
#define LSH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lsh_status {
  LSH_OK = 0,
  LSH_ERR_INVALID_ARG = 1, /* null required pointer, bad flag or parameter */
  LSH_ERR_SHAPE = 2,       /* size out of range, L % chunk != 0, odd n_buckets */
  LSH_ERR_DTYPE = 3,       /* unknown dtype code */
  LSH_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned */
  LSH_ERR_WORKSPACE = 5,   /* workspace missing or smaller than required */
  LSH_ERR_CUDA = 6,        /* a CUDA launch or runtime call failed */
  LSH_ERR_TIMEOUT = 7,     /* a device-side bounded wait ran out */
  LSH_ERR_UNSUPPORTED = 8  /* valid request that no kernel of this build serves */
} lsh_status;

typedef enum lsh_dtype { LSH_F32 = 0, LSH_BF16 = 1 } lsh_dtype;

/* Mask bits of lsh_chunk_attend. */
typedef enum lsh_mask {
  LSH_MASK_SELF = 1,    /* a slot does not see itself unless it is its only key */
  LSH_MASK_CAUSAL = 2,  /* a key after the query's original position is not admissible */
  LSH_MASK_BUCKET = 4,  /* a key in another bucket than the query's (this round) is not admissible */
  LSH_MASK_UNION = 8    /* lower each logit by log(#rounds sharing the bucket); needs LSH_MASK_BUCKET */
} lsh_mask;

/* Version of this ABI (incremented on any signature change). */
LSH_API int lsh_abi_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
LSH_API const char* lsh_status_string(int status);

/*
 * lsh_hash -- angular LSH of every shared query/key row, all rounds at once.
 * (Ultralytics glossary "Reformer", "Atencao LSH": bucket = position of the
 * largest value of [xR, -xR].)
 *
 *   qk        [B, H, L, D]  dtype          shared query/key rows
 *   R         [n_rounds, D, n_buckets/2] dtype   one random projection per round,
 *                                          shared by all batches and heads
 *   buckets   [B, H, n_rounds, L] int32    out: bucket in [0, n_buckets); entry k
 *                                          (< n_buckets/2) means +p_k was largest,
 *                                          k + n_buckets/2 means -p_k was
 *   near_tie  [B, H, n_rounds, L] uint8    out, nullable: 1 when the two largest
 *                                          values u1 >= u2 of [p, -p] satisfy
 *                                          u1 - u2 < 1e-5 * max(u1, 1e-30)
 *
 * p = x R is computed from the raw row (the argmax does not depend on the
 * row's length); products are exact and sums are fp32.  Exact ties go to the
 * lowest bucket index.  Requires n_buckets even, 2 <= n_buckets <= 65536,
 * D % 8 == 0, 8 <= D <= 256.
 */
LSH_API lsh_status lsh_hash(const void* qk, int dtype, int B, int H, int L, int D,
                    const void* R, int n_rounds, int n_buckets,
                    int32_t* buckets, uint8_t* near_tie, void* stream);

/*
 * Bytes of scratch that lsh_sort_permute needs for these sizes (0 when none).
 */
LSH_API size_t lsh_sort_workspace_bytes(int B, int H, int L, int n_rounds, int n_buckets);

/*
 * lsh_sort_permute -- stable sort of each (b, h, round) segment by the key
 * (bucket, position), and an optional gather of the sorted rows.
 * (twgreatdaily ICLR 2020 Reformer article, "1 LSH Attention": two-level
 * sort by bucket number and position inside the bucket.)
 *
 *   buckets    [B, H, n_rounds, L] int32   in, values in [0, n_buckets)
 *   perm       [B, H, n_rounds, L] int32   out: perm[s] = original position of
 *                                          sorted slot s
 *   inv        [B, H, n_rounds, L] int32   out, nullable: inv[perm[s]] = s
 *   qk, v      [B, H, L, D] dtype          in, nullable (both or neither): rows
 *                                          to gather in sorted order
 *   qk_sorted, v_sorted [B, H, n_rounds, L, D] dtype  out, nullable with qk/v:
 *                                          qk_sorted[..., s, :] = qk[..., perm[s], :]
 *   workspace  device scratch of at least lsh_sort_workspace_bytes(...) bytes,
 *              contents undefined on entry and on exit
 *
 * A bucket id outside [0, n_buckets) is a caller error: the kernels skip that
 * element, leave the slot it would have filled unwritten, and record
 * LSH_ERR_INVALID_ARG in the device status word (lsh_get_device_status).
 */
LSH_API lsh_status lsh_sort_permute(const int32_t* buckets, int B, int H, int L, int n_rounds,
                            int n_buckets, int32_t* perm, int32_t* inv,
                            const void* qk, const void* v, int dtype, int D,
                            void* qk_sorted, void* v_sorted,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * lsh_sort_permute_noalloc -- lsh_sort_permute (without the optional row
 * gather) for callers that cannot hand the library any scratch memory.
 * The pages have no counterpart of this call; it exists for this library's
 * users only.
 *
 * Some callers cannot allocate device memory while they run: a plugin that a
 * host application gives only its input and output buffers, a process whose
 * device memory another framework's pool has already reserved, or a code path
 * that must not pay cudaMalloc's implicit synchronisation.  This entry point
 * takes no workspace and allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library call): its scratch is a 16 MiB array of static device
 * memory inside the library, which every GPU that loads the library holds
 * until the process exits.
 *
 *   buckets, perm, inv: as for lsh_sort_permute (inv nullable).
 *
 * Shapes with L <= 65536 and n_buckets <= 1024 (the 64K workload among them)
 * are sorted by one CTA per segment entirely in shared memory and touch the
 * array not at all.  Larger shapes run the radix sort (one counting pass per
 * 8-bit digit of the bucket id), which takes, with S = B*H*n_rounds segments,
 * S * 256 * ceil(L / 4096) counter words, at most S * 64 + S + 3 more, and, when
 * n_buckets > 256, 2 * S * L words for the first pass's ids and positions; the
 * call returns LSH_ERR_WORKSPACE, before any launch, when that exceeds the
 * array's 4 Mi words (16 MiB).  All other argument rules and errors are those
 * of lsh_sort_permute.
 *
 * The first call on a device that needs the array looks up its device
 * address (with that device current) and keeps it for the life of the
 * process, so make that first call before any stream capture, and do not use
 * this call after cudaDeviceReset (the kept address would be stale).  Every
 * call on a device shares the one array and leaves its contents behind; the
 * call clears what must start at zero itself.  Calls whose work overlaps on
 * the GPU (different streams, or graphs running at the same time) race on the
 * array: order them, for example on one stream.
 */
LSH_API lsh_status lsh_sort_permute_noalloc(const int32_t* buckets, int B, int H, int L,
                                            int n_rounds, int n_buckets, int32_t* perm,
                                            int32_t* inv, void* stream);

/*
 * lsh_chunk_attend -- attention of every sorted slot to its own chunk and the
 * previous chunk, per round, scattered back to original token order.
 * (twgreatdaily ICLR 2020 Reformer article, "1 LSH Attention": sum over the
 * admissible set divided by its partition function, masked keys, Q = K with
 * normalised keys, later chunk looks back one chunk; rdly.ru Reformer summary,
 * "Разделение на блоки": fixed-size blocks of the sorted sequence.)
 *
 *   qk, v      [B, H, L, D] dtype          in: shared query/key rows and values
 *   perm       [B, H, n_rounds, L] int32   in: from lsh_sort_permute
 *   buckets    [B, H, n_rounds, L] int32   in, nullable: from lsh_hash (by original
 *              position); required by LSH_MASK_BUCKET and LSH_MASK_UNION, else unread
 *   qk_sorted, v_sorted  nullable [B, H, n_rounds, L, D] dtype: when given, the
 *              rows are read in sorted order from them instead of through perm
 *   chunk      chunk length c, L % c == 0.  Chunk k = sorted slots
 *              [k c, (k+1) c); its queries see the slots of chunk k-1 (none
 *              for k = 0: no wrap-around) and of chunk k
 *   mask       bits of lsh_mask: LSH_MASK_SELF (1): a slot does not see itself
 *              unless it is its only key; LSH_MASK_CAUSAL (2): a key whose
 *              original position perm[t] is after the query's perm[s] is not
 *              admissible (the pages' character-level language model; the self
 *              rule then applies to what remains, so a query with no earlier key
 *              in its window sees only itself); LSH_MASK_BUCKET (4): a key whose
 *              bucket buckets[r][perm[t]] differs from the query's is not
 *              admissible (the article's admissible set: the query's own bucket,
 *              batched by chunks; self rule as for causal); LSH_MASK_UNION (8,
 *              only with 4): each admissible logit is lowered by log N, N = the
 *              number of rounds r' with buckets[r'][i] == buckets[r'][j] (the
 *              article's multi-round union: lsh_combine_rounds then counts each
 *              shared key once).  Every mask runs on the tensor-core path
 *              (UNION there for up to 8 rounds, with a stream-ordered scratch
 *              buffer of 16 bytes per token, cudaMallocAsync / cudaFreeAsync on
 *              `stream`, holding each token's buckets in all rounds as fp16
 *              codes; a bucket id outside [0, 30720) has no code and records
 *              LSH_ERR_UNSUPPORTED in the device status word, its pairs then
 *              counting no shared round) and on the CUDA-core path
 *   scale      logit scale; <= 0 selects 1/sqrt(D).  logit(s, t) =
 *              scale * qk[perm[s]] . qk[perm[t]] / ||qk[perm[t]]||
 *   out_rounds [B, H, n_rounds, L, D] out_dtype  out: per-round softmax-weighted
 *              values, at the original position perm[s]
 *   lse        [B, H, n_rounds, L] float   out: per-round log-sum-exp of the
 *              logits, at the original position
 *
 * A key row of zero length contributes logit 0.  Requires D % 8 == 0,
 * 8 <= D <= 256, 1 <= chunk <= L.
 */
LSH_API lsh_status lsh_chunk_attend(const void* qk, const void* v, int dtype, int B, int H, int L,
                            int D, int n_rounds, const int32_t* perm, const int32_t* buckets,
                            const void* qk_sorted, const void* v_sorted, int chunk,
                            int mask, float scale, void* out_rounds, int out_dtype,
                            float* lse, void* stream);

/*
 * lsh_combine_rounds -- merge the rounds of every query by their log-sum-exp
 * weights: out = sum_r exp(lse_r - LSE) o_r with LSE = log sum_r exp(lse_r).
 * (twgreatdaily ICLR 2020 Reformer article, "1 LSH Attention": several hash
 * rounds, each with its own admissible set; weighting by each round's
 * partition function gives the softmax over the union of the rounds' key sets
 * counted with multiplicity.)
 *
 *   out_rounds [B, H, n_rounds, L, D] in_dtype
 *   lse        [B, H, n_rounds, L] float
 *   out        [B, H, L, D] out_dtype       out
 *   lse_out    [B, H, L] float              out, nullable: LSE
 */
LSH_API lsh_status lsh_combine_rounds(const void* out_rounds, int in_dtype, const float* lse,
                              int B, int H, int L, int D, int n_rounds, void* out,
                              int out_dtype, float* lse_out, void* stream);

/*
 * lsh_chunk_attend_backward -- gradients of sum(dout * out) with respect to the
 * shared rows and the values, where out is lsh_combine_rounds' merge of
 * lsh_chunk_attend's rounds.  (Training through LSH attention recomputes from
 * the stored hash: twgreatdaily ICLR 2020 Reformer article, "1 LSH Attention";
 * Ultralytics glossary "Reformer", "Atencao LSH".)  The hash, the sort and the
 * masks are held fixed; per admissible pair (i, j) of every round, with
 * p~ = exp(logit - LSE_i):
 *     dv_j += p~ dout_i,  dz = p~ (dout_i . v_j - dout_i . out_i),
 *     dqk_i += scale dz k_j,  and through k_j = qk_j / ||qk_j|| the key side.
 *
 *   qk, v, perm, buckets, chunk, mask, scale   as given to lsh_chunk_attend
 *   out        [B, H, L, D] out_dtype   in: the merged output (lsh_combine_rounds)
 *   lse        [B, H, L] float          in: its LSE (lse_out of lsh_combine_rounds)
 *   dout       [B, H, L, D] out_dtype   in: gradient of the loss w.r.t. out
 *   dqk, dv    [B, H, L, D] float       out: overwritten (zeroed, then accumulated
 *                                       over the rounds in order; deterministic)
 *
 * Every mask runs.  bf16 rows with bf16 out / dout, D = 128, chunk = 64 and
 * L % 128 == 0 run on the tensor cores of sm_100 with every mask (the union
 * correction up to 8 rounds): a per-token pass (LSE, dout . out, key lengths)
 * into a stream-ordered scratch buffer of 16 bytes per token, with masks a
 * per-slot pass (bucket, and whether the window leaves the token alone) into
 * 4 bytes per token and round, with the union correction each token's buckets
 * in all rounds (16 bytes per token; bucket ids below 30720, as for
 * lsh_chunk_attend) (cudaMallocAsync / cudaFreeAsync on
 * `stream`; LSH_ERR_CUDA if they cannot be had), then one launch per round.
 * Everything else runs on the CUDA cores (one launch per round after zeroing
 * dqk / dv).  Both keep the rounds in order, so the
 * result is deterministic.  A key row of zero length takes the clamp's linear
 * branch (its gradient is scaled by 1e12).
 * Requires what lsh_chunk_attend requires and B * H <= 65535.
 */
LSH_API lsh_status lsh_chunk_attend_backward(const void* qk, const void* v, int dtype, int B, int H, int L,
                                     int D, int n_rounds, const int32_t* perm, const int32_t* buckets,
                                     int chunk, int mask, float scale, const void* out, const float* lse,
                                     const void* dout, int out_dtype, float* dqk, float* dv, void* stream);

/*
 * Synchronises `stream`, then returns and clears the current device's status
 * word (LSH_OK when no kernel recorded an error).  Returns LSH_ERR_CUDA if the
 * synchronisation itself fails.
 */
LSH_API lsh_status lsh_get_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LSH_ATTENTION_HASH_H */

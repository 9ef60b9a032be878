/*
 * engram.h -- C ABI of the B200 (sm_100a) Engram N-gram Embedding library.
 *
 * The operations are those of the Qwen3.8-Flash-Next Engram N-gram Embedding
 * ("ple" in the checkpoint config), NeMo AutoModel engram API page:
 *   class Qwen3_8_FlashNextNGramEmbedding      -- hash raw token IDs into the
 *        packed multi-head table and concatenate the looked-up rows;
 *   class Qwen3_8_FlashNextOwnerShardedEmbedding -- row lookup on a table held
 *        by one rank (process_group=None), and the owner-side accumulation of
 *        each row's gradient in the backward pass.
 * Here the whole table lives on one GPU; the library never communicates.
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers must point to device memory of the
 *     current CUDA device, owned by the caller. The library never allocates;
 *     scratch space is passed in by the caller (see engram_backward).
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *     The return code reports host-side argument checks and launch errors
 *     only; results are ready when the stream reaches the call's end.
 *   - Return codes: ENGRAM_OK, ENGRAM_EINVAL (argument rejected on the host,
 *     nothing launched), ENGRAM_ENOSPC (workspace too small, nothing
 *     launched), ENGRAM_ECUDA (a CUDA launch failed). engram_status_string
 *     names each one.
 *   - Faults found on the device (a row index outside the table, malformed
 *     cu_seqlens) never trap: the kernel skips the offending access, records
 *     a bit in a per-device error word, and carries on. Read and clear it
 *     with engram_get_device_error.
 */
#ifndef ENGRAM_B200_H
#define ENGRAM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ENGRAM_ABI_VERSION 2

#if defined(__GNUC__)
#define ENGRAM_API __attribute__((visibility("default")))
#else
#define ENGRAM_API
#endif

#define ENGRAM_MAX_NGRAM 4   /* largest supported ngram_size */
#define ENGRAM_MAX_HEADS 32  /* largest (ngram_size - 1) * heads_per_ngram */

/* return codes */
#define ENGRAM_OK 0
#define ENGRAM_EINVAL 1
#define ENGRAM_ENOSPC 2
#define ENGRAM_ECUDA 3

/* element types of tables and gradients */
#define ENGRAM_F32 0
#define ENGRAM_BF16 1
#define ENGRAM_F16 2

/* bits of the device error word */
#define ENGRAM_DEVERR_ROW_RANGE 1u   /* a row index outside [0, table_rows) */
#define ENGRAM_DEVERR_CU_SEQLENS 2u  /* cu_seqlens not non-decreasing from 0 to T */
#define ENGRAM_DEVERR_SORT_TIMEOUT 4u /* the backward sort's grid barrier gave up waiting
                                         (results of that call are invalid) */
#define ENGRAM_DEVERR_COPY_TIMEOUT 8u /* a bulk copy into shared memory did not complete in
                                         time (results of that call are invalid) */
#define ENGRAM_DEVERR_CAPACITY 16u   /* an owner received more lookups than the exchange's
                                         capacity; the extra ones were dropped */
/* Same type as cudaStream_t, without requiring the CUDA headers. */
typedef struct CUstream_st *engram_stream_t;

/*
 * Hash configuration: the constructor arguments of the page's
 * Qwen3_8_FlashNextNGramEmbedding (ngram_size, heads_per_ngram,
 * eos_token_id, layer_multipliers, ngram_heads_vocab_sizes,
 * ngram_heads_offsets) plus the table shape of
 * Qwen3_8_FlashNextEngramTableConfig (num_embeddings, embedding_dim).
 *   H = (ngram_size - 1) * heads_per_ngram heads; head h in group
 *   g = h / heads_per_ngram hashes the order-(g + 2) n-gram ending at each
 *   token. Only the first ngram_size multipliers and the first H moduli and
 *   offsets are read. Requirements (else ENGRAM_EINVAL):
 *   2 <= ngram_size <= ENGRAM_MAX_NGRAM, heads_per_ngram >= 1,
 *   H <= ENGRAM_MAX_HEADS, vocab_sizes[h] >= 1, offsets[h] >= 0,
 *   offsets[h] + vocab_sizes[h] <= table_rows <= 2^31, dim >= 1.
 *   fill_id is the raw ID read where a token lacks valid earlier context
 *   (the page's sentence on it is cut off; 0 is the documented default).
 */
typedef struct engram_params {
    int32_t ngram_size;                      /* N, page default 3 */
    int32_t heads_per_ngram;                 /* K, page default 8 */
    int64_t multipliers[ENGRAM_MAX_NGRAM];   /* signed int64, [N] */
    int64_t vocab_sizes[ENGRAM_MAX_HEADS];   /* prime modulus per head, [H] */
    int64_t offsets[ENGRAM_MAX_HEADS];       /* global row offset per head, [H] */
    int64_t fill_id;                         /* ID used for missing context */
    int64_t table_rows;                      /* padded rows R of the table */
    int32_t dim;                             /* row width D (160) */
    int32_t eos_id;                          /* raw EOS token ID (248044) */
} engram_params_t;

/*
 * engram_hash -- NGramEmbedding._hash_input_ids with _shift_right_after_eos.
 * For token t of sequence s (cu_seqlens[s] <= t < cu_seqlens[s+1]) let x_k be
 * the token k places back, or fill_id if that position lies before the
 * sequence start or an EOS lies at any of positions t-k .. t-1 (context
 * resets after EOS; an EOS keeps its own left context). The order-n mix is
 * XOR_{k<n} (x_k * multipliers[k]) in wrapping signed int64 arithmetic and
 *   out_idx[t, h] = offsets[h] + floor_mod(mix_{g+2}, vocab_sizes[h]).
 *   ids        device, int32 [T] raw token IDs (any value; negative IDs are
 *              sign-extended to int64 before the multiply)
 *   cu_seqlens device, int32 [nseq + 1], cu[0] = 0, non-decreasing, cu[nseq]
 *              = T; NULL means one sequence [0, T). A [B, S] batch is
 *              cu = {0, S, 2S, ..., B*S}. Malformed bounds set
 *              ENGRAM_DEVERR_CU_SEQLENS (memory safety is unaffected).
 *   T          tokens, 0 <= T < 2^31
 *   out_idx    device, int32 [T, H] row-major
 */
ENGRAM_API int engram_hash(const engram_params_t *params, const int32_t *ids,
                const int32_t *cu_seqlens, int32_t nseq, int64_t T,
                int32_t *out_idx, engram_stream_t stream);

/*
 * engram_gather -- NGramEmbedding._lookup_ngram_ids on a single-rank table:
 *   out[i, :] = table[idx[i], :] for 0 <= i < n, bit for bit.
 *   table  device, [table_rows, dim] of dtype, 16-byte aligned
 *   dtype  ENGRAM_F32 | ENGRAM_BF16 | ENGRAM_F16; dim * sizeof(dtype) must be
 *          a multiple of 16 bytes
 *   idx    device, int32 [n]
 *   out    device, [n, dim] of dtype, 16-byte aligned
 * A negative index marks an absent lookup (the padding of a fixed-capacity
 * exchange): its output row is zero. An index >= table_rows also writes a zero
 * row and sets ENGRAM_DEVERR_ROW_RANGE.
 */
ENGRAM_API int engram_gather(const void *table, int32_t dtype, int64_t table_rows, int32_t dim,
                  const int32_t *idx, int64_t n, void *out, engram_stream_t stream);

/*
 * engram_hash_gather -- NGramEmbedding.forward: hash and lookup fused in one
 * kernel. out is [T, H, dim] of dtype (= [T, H * dim], heads concatenated in
 * head order: bigram heads first). out_idx may be NULL; if given it receives
 * the [T, H] row indices exactly as engram_hash writes them (the backward
 * needs them). Table requirements as engram_gather, table_rows and dim taken
 * from params.
 */
ENGRAM_API int engram_hash_gather(const engram_params_t *params, const int32_t *ids,
                       const int32_t *cu_seqlens, int32_t nseq, int64_t T,
                       const void *table, int32_t dtype, int32_t *out_idx,
                       void *out, engram_stream_t stream);

/*
 * engram_hash_gather_slice -- NGramEmbedding._forward_global_slice: hash the
 * complete stream but look up only positions [start, end) of every row, so
 * the earlier tokens and the EOS / sequence resets that a slice boundary cuts
 * off still shape the slice's first tokens (the page hashes the replicated
 * global IDs for this reason when context parallelism shards the sequence).
 *   ids, cu_seqlens, nseq, T  the whole stream, as for engram_hash
 *   row_len    tokens per row of a [T / row_len, row_len] batch (T must be a
 *              multiple); 0 means one row of T tokens
 *   start, end 0 <= start <= end <= row length
 *   out_idx    device, int32 [T / row_len, end - start, H] (may be NULL)
 *   out        device, [T / row_len, end - start, H * dim] of dtype
 * Equal to engram_hash_gather over the whole stream followed by taking
 * positions [start, end) of every row, without computing the rest.
 */
ENGRAM_API int engram_hash_gather_slice(const engram_params_t *params, const int32_t *ids,
                                        const int32_t *cu_seqlens, int32_t nseq, int64_t T,
                                        int64_t row_len, int64_t start, int64_t end,
                                        const void *table, int32_t dtype, int32_t *out_idx,
                                        void *out, engram_stream_t stream);

/*
 * engram_backward_workspace_size -- bytes of scratch engram_backward needs for
 * n lookups into a table of table_rows rows of width dim, on the current
 * device (the size depends on its SM count).
 */
ENGRAM_API int engram_backward_workspace_size(int64_t n, int64_t table_rows, int32_t dim,
                                   size_t *bytes);

/*
 * engram_backward -- gradient of the lookup with respect to the table, in
 * compact form (the owner-side row-gradient accumulation of the page's
 * OwnerShardedEmbedding; no dense [table_rows, dim] gradient is formed):
 *   uniq_rows[u]    = the u-th distinct value of idx[0..n), ascending
 *   row_grads[u, :] = sum over j with idx[j] == uniq_rows[u] of dout[j, :],
 *                     accumulated in fp64 and rounded once to fp32 (no
 *                     atomics; deterministic for a given device type)
 *   *num_unique     = U, the number of distinct rows
 *   idx        device, int32 [n], 0 <= n < 2^31; a negative value marks an
 *              absent lookup (the padding of a fixed-capacity exchange), left
 *              out of the rows and sums; values >= table_rows set
 *              ENGRAM_DEVERR_ROW_RANGE (results are then unspecified, memory
 *              accesses stay in bounds)
 *   dout       device, [n, dim] of dtype, 16-byte aligned; dim % 8 == 0 and
 *              dim <= 512
 *   uniq_rows  device, int32, capacity n
 *   row_grads  device, fp32 [n, dim] capacity, 16-byte aligned
 *   num_unique device, int32 scalar
 *   workspace  device, >= engram_backward_workspace_size bytes, 256-byte
 *              aligned; contents on entry are ignored
 * engram_backward = engram_backward_sort followed by engram_backward_reduce
 * with the same n, table_rows, dim and workspace.
 */
ENGRAM_API int engram_backward(const int32_t *idx, int64_t n, int64_t table_rows, int32_t dim,
                    const void *dout, int32_t dtype, int32_t *uniq_rows,
                    float *row_grads, int32_t *num_unique, void *workspace,
                    size_t workspace_bytes, engram_stream_t stream);

/* First stage: stable LSD radix sort of the (idx[j], j) pairs into the workspace.
 * One cooperative launch where the device supports it, else two launches per
 * radix pass; ENGRAM_SORT_SEPARATE_LAUNCHES=1 in the environment (read once per
 * process) forces the second form. Both give the same result. */
ENGRAM_API int engram_backward_sort(const int32_t *idx, int64_t n, int64_t table_rows, int32_t dim,
                         void *workspace, size_t workspace_bytes, engram_stream_t stream);

/* Second stage: distinct rows and segmented fp32 sums from the sorted pairs
 * that engram_backward_sort (or engram_backward_sort_heads) left in the
 * workspace. */
ENGRAM_API int engram_backward_reduce(int64_t n, int64_t table_rows, int32_t dim, const void *dout,
                           int32_t dtype, int32_t *uniq_rows, float *row_grads,
                           int32_t *num_unique, void *workspace, size_t workspace_bytes,
                           engram_stream_t stream);

/*
 * engram_backward_heads -- engram_backward for the lookups the hash produced
 * (engram API page, Qwen3_8_FlashNextNGramEmbedding._hash_input_ids and the
 * owner-side gradient accumulation of Qwen3_8_FlashNextOwnerShardedEmbedding),
 * with the same results, computed faster by using their structure: lookup
 * j = t * H + h of token t and head h lies in head h's slice
 * [offsets[h], offsets[h] + vocab_sizes[h]) of the table, and the heads'
 * slices ascend without overlapping. The sort then orders each head's T
 * lookups by row - offsets[h] (bits(vocab_sizes[h] - 1) bits: 25 on the
 * page's table, against 29 for the whole row, so 3 radix passes instead of 4)
 * and lays the heads out in order.
 *   params     the hash's parameters (H = (ngram_size - 1) * heads_per_ngram
 *              heads, table_rows, dim)
 *   idx        device, int32 [T, H] as engram_hash / engram_hash_gather wrote
 *              it; a value outside its head's slice sets
 *              ENGRAM_DEVERR_ROW_RANGE (results are then unspecified, memory
 *              accesses stay in bounds)
 *   T          tokens, n = T * H < 2^31
 *   dout, dtype, uniq_rows, row_grads, num_unique   as engram_backward with
 *              n = T * H lookups of width params->dim
 *   workspace  >= engram_backward_workspace_size(T * H, params->table_rows,
 *              params->dim) bytes, 256-byte aligned
 * Parameters whose slices do not ascend disjointly inside the table are
 * sorted as engram_backward sorts (same results).
 * engram_backward_heads = engram_backward_sort_heads followed by
 * engram_backward_reduce(T * H, params->table_rows, params->dim, ...) with the
 * same workspace.
 */
ENGRAM_API int engram_backward_heads(const engram_params_t *params, const int32_t *idx,
                                     int64_t T, const void *dout, int32_t dtype,
                                     int32_t *uniq_rows, float *row_grads, int32_t *num_unique,
                                     void *workspace, size_t workspace_bytes,
                                     engram_stream_t stream);

/* First stage of engram_backward_heads: the sort by head into the workspace
 * (one cooperative launch, or two launches per pass as engram_backward_sort). */
ENGRAM_API int engram_backward_sort_heads(const engram_params_t *params, const int32_t *idx,
                                          int64_t T, void *workspace, size_t workspace_bytes,
                                          engram_stream_t stream);

/* Size of the library's own device scratch array used by engram_backward_noalloc. */
#define ENGRAM_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20) /* 32 MiB per device */

/*
 * engram_backward_noalloc -- engram_backward for callers that cannot allocate
 * device memory: a plugin or kernel library inside a host application that
 * owns all device memory and offers no workspace hook, or a latency-critical
 * path that must not call cudaMalloc (which may synchronise the device). The
 * pages describe no such entry point; it is a convenience of this library.
 *
 * Same arguments and results as engram_backward, without the workspace: the
 * scratch lives in one file-scope device array of ENGRAM_NOALLOC_SCRATCH_BYTES
 * inside the library. Every GPU that loads the library holds that array until
 * the process exits. The call allocates nothing (no cudaMalloc, no cudaFree).
 *   - Sizes whose workspace (engram_backward_workspace_size) exceeds
 *     ENGRAM_NOALLOC_SCRATCH_BYTES are rejected with ENGRAM_ENOSPC before
 *     anything is launched.
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress); make that first call before any stream
 *     capture on the device.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (each call clears what must start at zero). Calls that overlap
 *     on the GPU -- on different streams, or from several host threads --
 *     race on it; serialise them, e.g. on one stream.
 */
ENGRAM_API int engram_backward_noalloc(const int32_t *idx, int64_t n, int64_t table_rows,
                                       int32_t dim, const void *dout, int32_t dtype,
                                       int32_t *uniq_rows, float *row_grads,
                                       int32_t *num_unique, engram_stream_t stream);

/* ------------------------------------------------------------------------
 * PLE layer tail: the consumer of the embedding inside
 * Qwen3_8_FlashNextPLELayer (engram page), after its key/value projections.
 * The page lists a branch-local Gemma RMS norm (norm_conv, and norm_key /
 * norm_query of the same kind: Qwen3_8_FlashNextGroupedRMSNorm, layers page)
 * and a causal depthwise convolution of width conv_kernel_size = 4 and
 * dilation short_conv_dilation = ngram_size = 3 with zero history
 * (_causal_short_conv; its context-parallel halo is (4 - 1) * 3 = 9 tokens).
 * The page prints neither an activation nor a residual for the convolution;
 * the Engram paper it cites applies x + SiLU(conv(norm(x))), which the
 * ENGRAM_CONV_* flags select step by step.
 * ------------------------------------------------------------------------ */

#define ENGRAM_CONV_NORM 1u     /* normalise each branch slice before the convolution */
#define ENGRAM_CONV_SILU 2u     /* y * sigmoid(y) after the convolution */
#define ENGRAM_CONV_RESIDUAL 4u /* add the (unnormalised) input */

typedef struct engram_conv_params {
    int32_t channels;     /* C = hc_count * hidden_size (page: 4 * 2560) */
    int32_t group_size;   /* G = hidden_size: features normalised together; C % G == 0,
                             G % 8 == 0, G <= 4096 */
    int32_t kernel_size;  /* K, 1 .. 8 (page: 4) */
    int32_t dilation;     /* d >= 1 (page: ngram_size = 3) */
    float eps;            /* rms_norm_eps (page default 1e-6), >= 0 */
    uint32_t flags;       /* ENGRAM_CONV_* bits */
    int32_t weight_dtype; /* ENGRAM_F32 | ENGRAM_BF16 | ENGRAM_F16 of the weights */
    int32_t reserved;     /* must be 0 */
} engram_conv_params_t;

/*
 * engram_ple_short_conv -- over x = [T, C] (C / G branch slices of G
 * features per token), for every token t of sequence s and channel c:
 *   n[t, c] = x[t, c] * rsqrt(mean over c's slice of x[t, .]^2 + eps)
 *             * (1 + norm_weight[c])        (ENGRAM_CONV_NORM; else n = x)
 *   y[t, c] = conv_bias[c] + sum over k < K with t - k*d >= cu_seqlens[s] of
 *             conv_weight[c, K - 1 - k] * n[t - k*d, c]
 *   out     = y * sigmoid(y) (ENGRAM_CONV_SILU), then + x (ENGRAM_CONV_RESIDUAL)
 * computed in fp32 and rounded once to out_dtype.
 *   x           device, [T, C] of dtype (F32 | BF16 | F16), 16-byte aligned
 *   cu_seqlens  device, int32 [nseq + 1] as for engram_hash (NULL = one
 *               sequence): the convolution's history is zero before each start
 *   norm_weight device, [C] of weight_dtype (NULL = zeros; read only with
 *               ENGRAM_CONV_NORM) -- the additive Gemma scale
 *   conv_weight device, [C, K] of weight_dtype (the [C, 1, K] depthwise
 *               conv1d weight; its last tap meets the current token)
 *   conv_bias   device, [C] of weight_dtype, or NULL
 *   out         device, [T, C] of out_dtype (dtype or ENGRAM_F32), 16-byte
 *               aligned, not overlapping x
 * Limits (else ENGRAM_EINVAL): those of engram_conv_params_t; and unless
 * K <= 4 and G <= 2560 (the page's shape: any dilation), also
 * 4 * G * ((K - 1) * d + 4) + 1152 <= 227 KB of shared memory per block.
 */
ENGRAM_API int engram_ple_short_conv(const engram_conv_params_t *params, const void *x,
                                     int32_t dtype, const int32_t *cu_seqlens, int32_t nseq,
                                     int64_t T, const void *norm_weight,
                                     const void *conv_weight, const void *conv_bias,
                                     void *out, int32_t out_dtype, engram_stream_t stream);

/*
 * engram_ple_short_conv_backward -- gradients of engram_ple_short_conv's
 * output (same params, x, cu_seqlens and weights) for training the layer. The
 * pages print no backward; it is the chain rule through the forward's steps.
 * With xh = x * inv (inv the slice's rsqrt as above), s = 1 + norm_weight,
 * n = s * xh, and dout = dL/dout:
 *   dy      = dout * (sg + y * sg * (1 - sg)), sg = sigmoid(y)
 *             (ENGRAM_CONV_SILU; else dy = dout)
 *   dn[t]   = sum over k < K with t + k*d in t's sequence of
 *             conv_weight[c, K - 1 - k] * dy[t + k*d]
 *   dx      = inv * (s * dn - xh * mean over the slice of (s * dn * xh))
 *             (ENGRAM_CONV_NORM; else dx = dn), then + dout (ENGRAM_CONV_RESIDUAL)
 *   dconv_weight[c, K - 1 - k] = sum over t of dy[t + k*d] * n[t]   (same pairs)
 *   dconv_bias[c]   = sum over t of dy[t]
 *   dnorm_weight[c] = sum over t of dn[t] * xh[t]    (0 without ENGRAM_CONV_NORM)
 * computed in fp32; dx rounded once to grad_dtype, the weight gradients
 * summed per block and then over blocks in a fixed order (results do not
 * depend on timing).
 *   dout          device, [T, C] of grad_dtype (F32 | BF16 | F16), 16-byte aligned
 *   dx            device, [T, C] of grad_dtype, 16-byte aligned, overlapping
 *                 neither x nor dout
 *   dconv_weight  device, fp32 [C, K]
 *   dconv_bias    device, fp32 [C], or NULL (not wanted)
 *   dnorm_weight  device, fp32 [C], or NULL (not wanted)
 *   workspace     device, >= engram_ple_short_conv_backward_workspace_size
 *                 bytes, 16-byte aligned (per-block partial sums; overwritten)
 * Limits (else ENGRAM_EINVAL): those of engram_conv_params_t, K <= 4 and
 * G <= 2560 (every pair of element types fits). Two launches; T = 0 writes
 * zero weight gradients.
 */
ENGRAM_API int engram_ple_short_conv_backward(
    const engram_conv_params_t *params, const void *x, int32_t dtype,
    const int32_t *cu_seqlens, int32_t nseq, int64_t T, const void *norm_weight,
    const void *conv_weight, const void *conv_bias, const void *dout, int32_t grad_dtype,
    void *dx, float *dnorm_weight, float *dconv_weight, float *dconv_bias, void *workspace,
    size_t workspace_bytes, engram_stream_t stream);

/*
 * engram_ple_short_conv_save -- engram_ple_short_conv that also keeps what
 * its backward needs from the norm, as an autograd norm keeps its rstd:
 *   inv_rms  device, fp32 [T, C / G], 4-byte aligned, overlapping neither x
 *            nor out: inv of every token's branch slices (ENGRAM_CONV_NORM
 *            required, else ENGRAM_EINVAL); NULL keeps nothing (then this is
 *            engram_ple_short_conv)
 * Same arguments, limits and output otherwise; saving changes no output bit.
 */
ENGRAM_API int engram_ple_short_conv_save(const engram_conv_params_t *params, const void *x,
                                          int32_t dtype, const int32_t *cu_seqlens,
                                          int32_t nseq, int64_t T, const void *norm_weight,
                                          const void *conv_weight, const void *conv_bias,
                                          void *out, int32_t out_dtype, float *inv_rms,
                                          engram_stream_t stream);

/*
 * engram_ple_short_conv_backward_saved -- engram_ple_short_conv_backward
 * given the inv_rms [T, C / G] that engram_ple_short_conv_save wrote for the
 * same x and params (the backward then skips computing it; it does not
 * check the values; 4-byte aligned). ENGRAM_CONV_NORM required, else
 * ENGRAM_EINVAL; NULL computes them (then this is
 * engram_ple_short_conv_backward). Same arguments, limits, workspace and
 * outputs otherwise; the results differ from the computing form only by
 * rounding (the saved values were summed in another order).
 */
ENGRAM_API int engram_ple_short_conv_backward_saved(
    const engram_conv_params_t *params, const void *x, int32_t dtype,
    const int32_t *cu_seqlens, int32_t nseq, int64_t T, const void *norm_weight,
    const void *conv_weight, const void *conv_bias, const float *inv_rms, const void *dout,
    int32_t grad_dtype, void *dx, float *dnorm_weight, float *dconv_weight, float *dconv_bias,
    void *workspace, size_t workspace_bytes, engram_stream_t stream);

/* Workspace bytes engram_ple_short_conv_backward needs for T tokens on the
 * current device (it depends on the device's multiprocessor count). */
ENGRAM_API int engram_ple_short_conv_backward_workspace_size(
    const engram_conv_params_t *params, int64_t T, size_t *bytes);

/*
 * engram_grouped_rms_norm -- Qwen3_8_FlashNextGroupedRMSNorm.forward over
 * `rows` rows of `channels` features: every group of group_size consecutive
 * features is normalised on its own,
 *   out[r, c] = x[r, c] * rsqrt(mean over c's group of x[r, .]^2 + eps)
 *               * (1 + weight[c])
 * in fp32, rounded once to out_dtype (dtype or ENGRAM_F32). weight [channels]
 * of weight_dtype, NULL = zeros (the page's reset value). out may be x itself
 * (same dtype). Limits: channels % group_size == 0, group_size % 8 == 0,
 * group_size <= 4096; x and out 16-byte aligned.
 */
ENGRAM_API int engram_grouped_rms_norm(const void *x, int32_t dtype, int64_t rows,
                                       int32_t channels, int32_t group_size,
                                       const void *weight, int32_t weight_dtype, float eps,
                                       void *out, int32_t out_dtype, engram_stream_t stream);

/* ------------------------------------------------------------------------
 * Optimizer step on the rows a backward produced. The pages say that the
 * owner stores and updates each row's gradient and that the Engram table
 * carries optimizer tensors in the checkpoint; they name no formula. This is
 * AdamW with per-row moments, applied lazily (only the listed rows change)
 * with the step count global to the table.
 * ------------------------------------------------------------------------ */

typedef struct engram_adam_params {
    float lr;            /* learning rate, >= 0 */
    float beta1, beta2;  /* in [0, 1) */
    float eps;           /* >= 0 */
    float weight_decay;  /* decoupled decay, >= 0 */
    int32_t reserved;    /* must be 0 */
    int64_t step;        /* 1 for the first update */
} engram_adam_params_t;

/*
 * engram_sparse_adam -- for u < U = min(*num_unique, max_rows), row
 * r = uniq_rows[u], gradient g = row_grads[u, :]:
 *   p[r] *= 1 - lr * weight_decay
 *   m[r]  = beta1 * m[r] + (1 - beta1) * g
 *   v[r]  = beta2 * v[r] + (1 - beta2) * g^2
 *   p[r] -= lr / (1 - beta1^step) * m[r] / (sqrt(v[r]) / sqrt(1 - beta2^step) + eps)
 * in fp32, p rounded once to dtype. Other rows are untouched.
 *   table      device, [table_rows, dim] of dtype (F32 | BF16 | F16), updated in
 *              place; 16-byte aligned (F32) or 8-byte aligned (BF16 / F16)
 *   exp_avg, exp_avg_sq  device, fp32 [table_rows, dim], 16-byte aligned, updated
 *   uniq_rows  device, int32 [>= U], distinct rows (the backward's output);
 *              a row outside the table is skipped and sets ENGRAM_DEVERR_ROW_RANGE
 *   row_grads  device, fp32 [>= U, dim], 16-byte aligned
 *   num_unique device, int32 scalar (read on the device: no host round trip
 *              after engram_backward)
 *   max_rows   capacity of uniq_rows / row_grads
 * dim % 4 == 0. Rows listed twice race (the backward lists each row once).
 */
ENGRAM_API int engram_sparse_adam(const engram_adam_params_t *params, void *table,
                                  int32_t dtype, int64_t table_rows, int32_t dim,
                                  float *exp_avg, float *exp_avg_sq,
                                  const int32_t *uniq_rows, const float *row_grads,
                                  const int32_t *num_unique, int64_t max_rows,
                                  engram_stream_t stream);

/* ------------------------------------------------------------------------
 * Owner-sharded table (Qwen3_8_FlashNextOwnerShardedEmbedding, engram page):
 * rank r of an owner group of `owners` ranks holds rows
 * [r * rows_per_owner, (r + 1) * rows_per_owner) of the table. A requesting
 * rank groups its lookups by owner, sends the owner-local rows in the first
 * All-to-All, the owners look them up (engram_gather on their shard), and the
 * second All-to-All brings the values back in the same grouping; in the
 * backward the row gradients travel the reverse way and only the owner
 * accumulates them (engram_backward on its shard). The collectives themselves
 * are the caller's (NCCL through torch.distributed in the Python package);
 * this call is the routing step on the requesting rank.
 * ------------------------------------------------------------------------ */

/*
 * engram_owner_bucket -- stable grouping of n lookups by owner
 * o = rows[i] / rows_per_owner. For the lookup i placed at grouped position p
 * (owners in ascending order, each owner's lookups in ascending i):
 *   send_rows[p] = rows[i] - o * rows_per_owner   (owner-local row)
 *   src_pos[p]   = i
 *   dst_pos[i]   = p
 *   counts[o]    = lookups of owner o (device, int32 [owners])
 * so engram_gather(values, dst_pos) restores request order from values that
 * came back grouped, and engram_gather(dout, src_pos) groups the gradients.
 * A row outside [0, owners * rows_per_owner) goes to the last owner with
 * local row -1 (which that owner's lookup rejects) and sets
 * ENGRAM_DEVERR_ROW_RANGE.
 *   rows       device, int32 [n] (e.g. engram_hash's [T, H] output)
 *   send_rows, src_pos, dst_pos  device, int32 [n], not overlapping rows
 *   workspace  device, >= engram_owner_bucket_workspace_size bytes
 * Limits: 1 <= owners <= 256, rows_per_owner >= 1, 0 <= n < 2^31. Three
 * launches.
 */
ENGRAM_API int engram_owner_bucket(const int32_t *rows, int64_t n, int64_t rows_per_owner,
                                   int32_t owners, int32_t *send_rows, int32_t *src_pos,
                                   int32_t *dst_pos, int32_t *counts, void *workspace,
                                   size_t workspace_bytes, engram_stream_t stream);

ENGRAM_API int engram_owner_bucket_workspace_size(int64_t n, int32_t owners, size_t *bytes);

/*
 * engram_owner_bucket_padded -- engram_owner_bucket into the fixed-capacity
 * layout of the engram API page's _FixedCapacityAllToAll /
 * _fixed_capacity_all_to_all: every owner gets a segment of `capacity` slots,
 * agreed ahead of time, so that both exchanges are equal-split all-to-alls
 * whose sizes never depend on the data and the step needs no host
 * synchronisation (it can be captured in a CUDA graph).
 *   send_rows[o * capacity + k], src_pos[o * capacity + k]
 *              owner o's k-th lookup (as engram_owner_bucket) for
 *              k < counts[o]; -1 in the padding slots k >= counts[o]
 *   dst_pos[i] o * capacity + k for lookup i, or -1 if owner o already had
 *              `capacity` lookups (the lookup is dropped and
 *              ENGRAM_DEVERR_CAPACITY is set)
 *   counts[o]  min(lookups of owner o, capacity)
 * The lookup (engram_gather) and the backward (engram_backward) treat the -1
 * entries as absent: zero rows, left out of the gradient. capacity = n never
 * drops a lookup. send_rows and src_pos hold owners * capacity int32 each
 * (owners * capacity < 2^31); workspace as engram_owner_bucket.
 */
ENGRAM_API int engram_owner_bucket_padded(const int32_t *rows, int64_t n,
                                          int64_t rows_per_owner, int32_t owners,
                                          int64_t capacity, int32_t *send_rows,
                                          int32_t *src_pos, int32_t *dst_pos, int32_t *counts,
                                          void *workspace, size_t workspace_bytes,
                                          engram_stream_t stream);

/*
 * engram_get_device_error -- copy the current device's error word
 * (ENGRAM_DEVERR_* bits set since the last call) into *flags and clear it.
 * Synchronises `stream`. Calls on several streams share one word.
 */
ENGRAM_API int engram_get_device_error(uint32_t *flags, engram_stream_t stream);

/* Static description of a return code. */
ENGRAM_API const char *engram_status_string(int status);

/* ENGRAM_ABI_VERSION of the loaded library. */
ENGRAM_API int engram_abi_version(void);

/* sizeof(engram_params_t) as compiled into the library (binding layout check). */
ENGRAM_API size_t engram_params_size(void);

/* Number of kernels this library has launched in this process. */
ENGRAM_API uint64_t engram_launch_count(void);

/*
 * Host-side check of the device modular reduction: floor_mod(a, m) for
 * 1 <= m < 2^32, computed on the CPU by the same Barrett routine the kernels
 * use (result in [0, m); 0 with ENGRAM_EINVAL in *status otherwise).
 */
ENGRAM_API int64_t engram_host_floor_mod(int64_t a, int64_t m, int *status);

#ifdef __cplusplus
}
#endif

#endif /* ENGRAM_B200_H */

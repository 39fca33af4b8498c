/*
 * dspark_markov.h -- C ABI of the B200 (sm_100a) VanillaMarkov transition-bias head.
 *
 * The head (markov_head.py, the vendored DSpark-style low-rank Markov sequential
 * head: module docstring "WHAT THIS IS" and class VanillaMarkov) adds a
 * rank-r bias that depends only on the previous token to a parallel block
 * drafter's base logits:
 *
 *     corrected_k[v] = U_k[v] + B(x_{k-1}, v),   B(x, v) = sum_j W1[x, j] * W2[v, j]
 *
 * W1 is an embedding table and W2 the weight of a bias-free Linear(r, V); both
 * are stored [V, r] row-major, exactly as the two PyTorch modules store them.
 *
 * Conventions shared by every entry point:
 *   - Every buffer is caller-owned DEVICE memory on the current CUDA device,
 *     contiguous row-major. The library never frees or keeps a caller pointer
 *     beyond the call.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and the call returns without synchronising. Results are valid
 *     once the stream has reached that point.
 *   - The return value is a DSPARK_* code. Argument errors are detected on the
 *     host before anything is enqueued. Errors found on the device (a token id
 *     outside [0, V), a bounded wait that ran out) never trap: they are OR-ed
 *     into a per-device status word read by dspark_markov_get_status().
 *   - logits_dtype / weight_dtype are DSPARK_DTYPE_* codes. Sums are
 *     accumulated in fp32 and the corrected logit is rounded once (round to
 *     nearest even) to the logits dtype.
 *   - The library keeps a small per-device workspace (status word, reduction
 *     keys and a barrier counter for the sampler), allocated on first use and
 *     grown when a larger sampler call needs it. Calls that use it must not
 *     run concurrently on one device (issue them on one stream).
 */
#ifndef DSPARK_MARKOV_H
#define DSPARK_MARKOV_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define DSPARK_OK 0
#define DSPARK_ERR_INVALID_ARG 1 /* null pointer, non-positive size, rank <= 0, NaN temperature, ... */
#define DSPARK_ERR_UNSUPPORTED 2 /* dtype pair or shape this build does not handle */
#define DSPARK_ERR_CUDA 3        /* a CUDA runtime call or kernel launch failed */

/* Bits of the device status word (dspark_markov_get_status). */
#define DSPARK_STATUS_TOKEN_RANGE 1u /* a token id was outside [0, V); its bias was taken as 0 */
#define DSPARK_STATUS_TIMEOUT 2u     /* a bounded device-side wait ran out; outputs are invalid */

/* Element types. */
#define DSPARK_DTYPE_FP32 0
#define DSPARK_DTYPE_BF16 1

/* Kernel selection (dspark_markov_set_algo). */
#define DSPARK_ALGO_AUTO 0         /* tensor-core kernels where the shape allows, else generic */
#define DSPARK_ALGO_GENERIC 1      /* CUDA-core kernels for any shape and dtype */
#define DSPARK_ALGO_TENSOR_CORE 2  /* tcgen05 kernels only; other shapes return DSPARK_ERR_UNSUPPORTED */

/*
 * Teacher-forced corrected logits for every position at once
 * (VanillaMarkov.apply_block_logits; markov_head API docs: "apply_block_logits").
 *
 *   base_logits    [rows, vocab] logits_dtype. The pages' [B, num_blocks, block_size, V]
 *                  or (R, M, V) layouts flatten to rows = product of the leading dims.
 *   out            [rows, vocab] logits_dtype. May equal base_logits (in place).
 *   prev_token_ids [rows] int64: the teacher-forced previous token of each row.
 *   w1, w2         [vocab, rank] weight_dtype (embedding table; Linear(rank, vocab) weight).
 *   rank           > 0 (the head requires markov_rank > 0).
 *
 * rows == 0 is OK and enqueues nothing (the pages return the input itself when
 * it is empty). The vanilla head ignores hidden states, so none are passed.
 * Supported dtype pairs: (fp32, fp32), (bf16, bf16), (fp32 logits, bf16 weights),
 * (bf16 logits, fp32 weights).
 */
int dspark_markov_apply_block_logits(const void* base_logits, void* out, const int64_t* prev_token_ids,
                                     int64_t rows, int64_t vocab, const void* w1, const void* w2, int32_t rank,
                                     int32_t logits_dtype, int32_t weight_dtype, void* stream);

/*
 * Gradients of the teacher-forced apply, its train-time use
 * (markov_head.py, the vendored DSpark-style low-rank Markov head: "At TRAIN time
 * x_{k-1} is the teacher-forced ground-truth predecessor (apply_block_logits)").
 * With out = U + W1[x] W2^T and grad_out = dOut [rows, vocab]:
 *
 *     grad of base_logits = grad_out           (identity: nothing is computed)
 *     grad_w2[v, j] (+)= sum_i dOut[i, v] W1[x_i, j]
 *     grad_w1[x, j] (+)= sum over rows i with x_i = x of sum_v dOut[i, v] W2[v, j]
 *
 *   grad_out        [rows, vocab] logits_dtype; prev_token_ids [rows] int64.
 *   w1, w2          [vocab, rank] weight_dtype (rank <= 1024).
 *   grad_w1/grad_w2 [vocab, rank] fp32, caller-owned; either may be NULL (not wanted).
 *   accumulate      nonzero: add into the buffers (as autograd accumulates .grad);
 *                   zero: overwrite them.
 *
 * Sums are accumulated in fp32 (grad_w1 with atomics, so the order of its
 * additions varies from run to run). A row whose id is outside [0, vocab)
 * contributes nothing and sets DSPARK_STATUS_TOKEN_RANGE.
 *
 * bf16 grad_out with bf16 weights, vocab % 8 == 0, rank in {64, 128, 192, 256}
 * and 16-byte aligned pointers run on the tensor cores (two launches: dW2, then
 * dW1); everything else on CUDA-core kernels. DSPARK_ALGO_TENSOR_CORE set by
 * dspark_markov_set_algo makes an unsupported call return
 * DSPARK_ERR_UNSUPPORTED; dspark_markov_last_algo reports 2 (tensor cores) or
 * 1 (CUDA cores).
 */
int dspark_markov_apply_block_logits_backward(const void* grad_out, const int64_t* prev_token_ids, int64_t rows,
                                              int64_t vocab, const void* w1, const void* w2, int32_t rank,
                                              float* grad_w1, float* grad_w2, int32_t accumulate,
                                              int32_t logits_dtype, int32_t weight_dtype, void* stream);

/*
 * Corrected logits with the base logits produced in the same pass (the step
 * before the head on the path: "U_k is the backbone's base logit
 * (lm_head(hidden_k))", module docstring of markov_head.py; the frozen
 * vocabulary head of DeepseekV41DSparkModel.compute_logits, weight
 * [vocab, hidden], FP32 result). For each row i with previous token
 * x = prev_token_ids[i]:
 *
 *     out[i, v] = round( sum_{j<hidden_dim} hidden[i, j] * lm_head[v, j]
 *                        + sum_{j<rank} W1[x, j] * W2[v, j] )
 *
 * one fp32 accumulation over both sums and one rounding (nearest even) to
 * out_dtype, so the base logits are never stored.
 *
 *   hidden          [rows, hidden_dim] weight_dtype, row-major.
 *   prev_token_ids  [rows] int64 (teacher-forced previous tokens).
 *   lm_head         [vocab, hidden_dim] weight_dtype (the LM head's weight).
 *   w1, w2          [vocab, rank] weight_dtype.
 *   out             [rows, vocab] out_dtype (DSPARK_DTYPE_FP32, as the pages'
 *                   compute_logits returns, or DSPARK_DTYPE_BF16), written.
 *
 * Supported: weight_dtype DSPARK_DTYPE_BF16; hidden_dim, rank and vocab
 * multiples of 8; every pointer 16-byte aligned; anything else returns
 * DSPARK_ERR_UNSUPPORTED (there is no other kernel for this entry). An id
 * outside [0, vocab) adds a zero bias for its row and sets
 * DSPARK_STATUS_TOKEN_RANGE. rows == 0 is OK and enqueues nothing.
 * Ownership and errors as for dspark_markov_apply_block_logits; `out` must
 * not overlap the inputs.
 */
int dspark_markov_fused_lm_head_logits(const void* hidden, const int64_t* prev_token_ids, int64_t rows,
                                       int64_t hidden_dim, int64_t vocab, const void* lm_head, const void* w1,
                                       const void* w2, int32_t rank, void* out, int32_t out_dtype,
                                       int32_t weight_dtype, void* stream);

/*
 * The transition bias alone, and its conditioning embeddings
 * (nemo_automodel.components.models.deepseek_v41.dspark,
 * _DeepseekV41DSparkMarkovHead.forward: "transition logits of shape [..., vocab]
 * and embeddings"). For each row i with token x = token_ids[i]:
 *
 *     transition_out[i, v] = round( sum_j W1[x, j] * W2[v, j] )   (weight_dtype)
 *     embeddings_out[i, j] = W1[x, j]                             (exact copy)
 *
 *   token_ids       [rows] int64 (the pages' [...] leading shape, flattened).
 *   w1, w2          [vocab, rank] weight_dtype.
 *   transition_out  [rows, vocab] weight_dtype, written.
 *   embeddings_out  [rows, rank] weight_dtype, written; may be NULL (not wanted).
 *
 * The sum is accumulated in fp32 and rounded once (nearest even). An id outside
 * [0, vocab) gives a zero bias row and a zero embedding row and sets
 * DSPARK_STATUS_TOKEN_RANGE. rows == 0 is OK and enqueues nothing.
 */
int dspark_markov_transition_logits(const int64_t* token_ids, int64_t rows, int64_t vocab, const void* w1,
                                    const void* w2, int32_t rank, void* transition_out, void* embeddings_out,
                                    int32_t weight_dtype, void* stream);

/*
 * Left-to-right sampling of B blocks of M positions
 * (VanillaMarkov.sample_block_tokens and _sample_tokens; markov_head API docs:
 * "sample_block_tokens").
 *
 *   base_logits          [batch, proposal_len, vocab] logits_dtype.
 *   first_prev_token_ids [batch] int64: the verified token before position 0.
 *   sampled_tokens       [batch, proposal_len] int64, written.
 *   corrected_logits     [batch, proposal_len, vocab] logits_dtype, written; the
 *                        values before any division by the temperature. Must
 *                        not overlap base_logits.
 *
 * Position k is corrected with the bias of the token chosen at k-1, and its own
 * choice feeds position k+1 on the device. temperature < 1e-5 means greedy:
 * the lowest index among the maxima of the ROUNDED corrected logits (NaN counts
 * as the largest value). Otherwise one draw from softmax(c / T) per (b, k), as
 * argmax_v(c_v / T + g_v) with Gumbel noise g = -log(-log u), u from
 * Philox4x32-10 (Salmon et al., SC'11) with key (seed lo, seed hi), counter
 * (v >> 2, k, b, 0), output word v & 3, and u = (2 * (word >> 9) + 1) * 2^-24.
 * proposal_len == 0 is OK and enqueues nothing. NaN temperature is
 * DSPARK_ERR_INVALID_ARG.
 */
int dspark_markov_sample_block(const void* base_logits, const int64_t* first_prev_token_ids, int64_t batch,
                               int64_t proposal_len, int64_t vocab, const void* w1, const void* w2, int32_t rank,
                               float temperature, uint64_t seed, int64_t* sampled_tokens, void* corrected_logits,
                               int32_t logits_dtype, int32_t weight_dtype, void* stream);

/*
 * dspark_markov_sample_block without any device allocation. The pages define
 * no counterpart: this is a library entry for callers that must not allocate
 * device memory during the call -- a serving loop whose memory is fully
 * reserved up front, a caller holding its own allocator's lock, or code on a
 * path where an allocation (or the implicit synchronisation cudaFree does)
 * would stall other streams. dspark_markov_sample_block keeps its reduction
 * keys and barrier counter in a workspace that it allocates on first use and
 * regrows for larger calls; this entry uses a fixed scratch in the library's
 * static device memory instead.
 *
 *   Arguments, layouts, ownership and results are those of
 *   dspark_markov_sample_block; the tensor-core sampler is always used (the
 *   process-wide DSPARK_ALGO_* choice does not apply).
 *   batch * proposal_len must not exceed DSPARK_NOALLOC_MAX_KEYS (8192, for
 *   64 KiB of scratch); larger calls return DSPARK_ERR_UNSUPPORTED, as do the
 *   shapes, dtypes and alignments the tensor-core sampler does not take
 *   (bf16 logits and weights, rank a multiple of 64 in [64, 256], vocab a
 *   multiple of 8, batch <= 256, 16-byte aligned buffers).
 *   The first call on each device looks up the scratch's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture. Every call clears the scratch's counter and
 *   keys with an asynchronous memset on `stream` and then launches one kernel.
 *   Device-side errors go to a status word in the scratch, which
 *   dspark_markov_get_status folds into the value it returns.
 *   There is one scratch per device: calls that overlap on one device (other
 *   streams or threads without ordering between them) race on it and give
 *   wrong results. Issue them on one stream or order them with events.
 */
#define DSPARK_NOALLOC_MAX_KEYS 8192
int dspark_markov_sample_block_noalloc(const void* base_logits, const int64_t* first_prev_token_ids, int64_t batch,
                                       int64_t proposal_len, int64_t vocab, const void* w1, const void* w2,
                                       int32_t rank, float temperature, uint64_t seed, int64_t* sampled_tokens,
                                       void* corrected_logits, int32_t logits_dtype, int32_t weight_dtype,
                                       void* stream);

/*
 * Synchronise `stream`, then read and clear the current device's status word
 * (DSPARK_STATUS_* bits) into *status_out. Not part of the hot path.
 */
int dspark_markov_get_status(void* stream, int32_t* status_out);

/* Text for a DSPARK_* return code. The string is static. */
const char* dspark_markov_strerror(int code);

/* Process-wide kernel selection (DSPARK_ALGO_*); returns the previous value. */
int32_t dspark_markov_set_algo(int32_t algo);

/* Number of kernels this library has launched in this process. */
int64_t dspark_markov_launch_count(void);

/*
 * Test hooks. `wait_limit_ns` bounds every device-side wait (0 restores the
 * default of about two seconds). `flags` bit 0 makes one CTA of the tensor-core
 * sampler skip its grid-barrier arrival, so that the others' bounded wait runs
 * out and reports DSPARK_STATUS_TIMEOUT; no GPU fault is involved.
 */
#define DSPARK_DEBUG_SKIP_BARRIER_ARRIVAL 1u
/* flags bit 1: the tensor-core apply uses 256-id units where they apply
 * (bf16 logits with a base, out != base_logits) instead of 128-id units.
 * flags bit 2: the tensor-core sampler uses the row layout (batch on the MMA's
 * M side) where it applies. flags bit 3: the tensor-core sampler uses the
 * tile layout (vocabulary ids on M) where it applies; bit 2 wins when both are
 * set. Without these bits each call takes the variant that measured fastest
 * on these shapes (row layout for temperature sampling, tile layout for
 * greedy decoding); every variant stays testable. */
#define DSPARK_DEBUG_APPLY_WIDE 2u
#define DSPARK_DEBUG_SAMPLE_ROWS 4u
#define DSPARK_DEBUG_SAMPLE_TILE 8u
int dspark_markov_set_debug(uint32_t flags, uint64_t wait_limit_ns);

/* Which kernel the last call on this thread selected: 0 none, 1 generic, 2 tensor core. */
int32_t dspark_markov_last_algo(void);

/*
 * Test hook: DSPARK_VARIANT_* bits naming the tensor-core kernel variants the
 * last call on this thread launched (0 when it launched none of them).
 *   DSPARK_VARIANT_BWD_RESIDENT_W1: the backward's dW2 kernel gathered every
 *     row's W1 row once into a resident shared-memory block (rows <= 8192 and
 *     the block fits beside three gradient stages), instead of once per stage.
 */
#define DSPARK_VARIANT_BWD_RESIDENT_W1 1
/*
 *   DSPARK_VARIANT_SAMPLE_ROWS: the tensor-core sampler ran with the batch on
 *     the MMA's M side and 256 vocabulary ids per MMA (batch <= 64; chosen for
 *     temperature > 0, by DSPARK_DEBUG_SAMPLE_ROWS, or where the tile layout
 *     does not fit; not under DSPARK_DEBUG_SAMPLE_TILE where the tile fits);
 *     otherwise it ran with vocabulary ids on M and the batch on N.
 */
#define DSPARK_VARIANT_SAMPLE_ROWS 2
/*
 *   DSPARK_VARIANT_APPLY_WIDE: the tensor-core apply ran with units of 128 rows
 *     x 256 ids (chosen by DSPARK_DEBUG_APPLY_WIDE); otherwise with 128 x 128.
 */
#define DSPARK_VARIANT_APPLY_WIDE 4
int32_t dspark_markov_last_variant(void);

/*
 * Test hook: out[i] = the Gumbel variate g = -log(-log u) that every sampler
 * kernel draws for the Philox output word words[i] (u = (2 (w >> 9) + 1) 2^-24),
 * computed by the same device function. words, out: n caller-owned device
 * elements. |g - exact| is below about 5e-6 for every word. n == 0 enqueues
 * nothing; n < 0 or a null buffer with n > 0 is DSPARK_ERR_INVALID_ARG.
 */
int dspark_markov_debug_gumbel(const uint32_t* words, float* out, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_MARKOV_H */

/*
 * uno.h — C ABI of the Uno draft-and-verify hot path on NVIDIA B200 (sm_100a).
 *
 * Three operations, each stated by the Uno pages:
 *   uno_gated_lora_linear  the row-gated LoRA projection (LoopUno project page, "How it
 *                          works" and "Setup / Recipe"; uno-qwen3-8B model card intro)
 *   uno_block_verify       lossless verification of a drafted block (LoopUno project page,
 *                          "How it works", "Training is self-distillation"; model card,
 *                          "Evaluation protocol")
 *   uno_tv_loss            the TV self-distillation loss and its gradient (LoopUno project
 *                          page, "Training is self-distillation")
 * and the block-noised copy that feeds the drafter and the student:
 *   uno_block_noise        noise mode random_uniform (LoopUno project page, "Training is
 *                          self-distillation"; model card, "Evaluation protocol")
 *
 * Conventions shared by every entry point
 *   - Pointers named as tensors are DEVICE pointers owned by the caller, row-major and
 *     contiguous, unless a comment says "host". The library never allocates, frees or
 *     keeps caller memory, and never synchronises the stream.
 *   - Scratch memory is a caller-supplied device `workspace` of at least the size the
 *     matching uno_*_workspace_size() reports (256-byte aligned). A workspace may be reused
 *     by later calls on the same stream, but two calls that may run at the same time need
 *     two workspaces.
 *   - Every call validates its arguments on the host before any launch and returns a
 *     uno_status; on error nothing is launched and no output is written. Errors are never
 *     signalled by a device trap. A call that returns UNO_OK has only been enqueued on
 *     `stream` (asynchronous); results are ready after the stream reaches that point.
 *   - uno_last_error_string() gives a readable reason for the calling thread's last
 *     failing call.
 *   - Device pointers must be 16-byte aligned (uno_block_noise: 4-byte aligned).
 *   - bf16 is IEEE-754 binary32 truncated to its upper 16 bits (1-8-7), stored as uint16.
 *
 * Kernel variants (environment, read at each call; every variant computes the same result
 * up to floating-point summation order, and the defaults are the fastest measured ones)
 *   UNO_LORA_CG=1|2          gated LoRA on single CTAs / CTA pairs (256-row tiles, cta_group::2)
 *   UNO_LORA_BN=64|128|256   gated LoRA output tile width (with UNO_LORA_CG=2: pair tile width)
 *   UNO_LORA_SPLITS=n        adapter product X A^T split over K into n bf16 partials of T
 *   UNO_LORA_KSPLIT=n        output tiles split over K into n fp32 partials
 *   UNO_LORA_EPI=rows        output tiles stored by lanes (no shared-memory staging)
 *   UNO_LORA_WIDE=0          one K slab per TMA load (default: two)
 *   UNO_LORA_COOP=0          gated LoRA launched without the cooperative attribute (for
 *                            profilers that run cooperative cluster launches as single CTAs)
 *   UNO_VERIFY_STREAM=warps|tma  top-k verify: per-segment streaming CTAs (register or bulk-copy fed)
 *   UNO_VERIFY_SEGMENTS=n    top-k verify with UNO_VERIFY_STREAM=warps: CTAs per row (1 to 8)
 *   UNO_VERIFY_TOPK=local|window  top-k verify on the cluster kernels
 *   UNO_VERIFY_PDL=0         top-k verify: the finish kernel launched after the streaming one ends
 *   UNO_VERIFY_FULL=generic  full-vocabulary verify: one CTA per item, fp64 exp per token;
 *                  =cluster  the cluster form or UNO_ERR_UNSUPPORTED
 *   UNO_VERIFY_FULL_CLUSTER=c  full-vocabulary cluster form: clusters of c CTAs
 *   UNO_VERIFY_LISTS=off     full-vocabulary verify without candidate lists
 *   UNO_VERIFY_ROW_CTAS=2    full-vocabulary row pass: two CTAs per SM
 *   UNO_TV_KERNEL=rows|teams TV loss: one CTA per row / two teams per CTA
 *   UNO_TV_CLUSTER=c         TV loss: clusters of c CTAs (1 to 8, or 16)
 *   UNO_TV_KEEP=0|1          TV loss: exp(student) recomputed / kept in shared memory
 * A workspace must be sized under the same settings as the call that uses it.
 */
#ifndef UNO_H
#define UNO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream). NULL is the legacy default stream. */
typedef struct CUstream_st* uno_stream_t;

typedef enum {
    UNO_OK = 0,
    UNO_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad scalar parameter */
    UNO_ERR_UNSUPPORTED = 2,   /* shape / dtype / alignment outside the supported limits */
    UNO_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed (see last error) */
    UNO_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up (device status word) */
    UNO_ERR_WORKSPACE = 5      /* workspace missing, too small or misaligned */
} uno_status;

typedef enum {
    UNO_BF16 = 0,
    UNO_F32 = 1
} uno_dtype;

/* Readable name of a status code (static storage). */
const char* uno_status_string(uno_status status);

/* Detail of the calling thread's last failing call ("" if none; thread-local storage). */
const char* uno_last_error_string(void);

/* ABI version of this library: major * 10000 + minor * 100 + patch. */
int uno_version(void);

/*
 * Device status word: kernels whose bounded waits time out record UNO_ERR_TIMEOUT there
 * instead of trapping; the CTA-pair gated LoRA kernel records UNO_ERR_UNSUPPORTED there
 * and does nothing when it finds itself launched without its two-CTA clusters. This call synchronises the current device, returns the word in
 * *code (UNO_OK if no kernel recorded anything since the last read) and clears it.
 * There is one word per device, shared by every stream and host thread that uses the
 * library on that device: a timeout recorded by any call since the last read is reported
 * to whichever caller reads first. Callers that run calls concurrently on several streams
 * learn that some call timed out, not which.
 */
uno_status uno_read_device_status(uint32_t* code);

/* ======================================================================================
 * Row-gated LoRA linear
 *
 *   Y = X W0^T + scale * diag(g) (X A^T) B^T
 *
 * The frozen base weight W0 serves every row; the rank-r adapter (A, B) is added only on
 * rows whose gate is non-zero (draft-noise rows; the seed / prefill / verify / AR rows
 * have gate 0). Source: LoopUno project page, "How it works" (one LoRA switched on only for
 * noise positions) and "Setup / Recipe" (gated LoRA, r=128, alpha=2048, all seven
 * projections, noise rows only); uno-qwen3-8B model card introduction (adapter applied
 * selectively on draft-noise rows).
 *
 *   x       [M, d_in]      activations, dtype
 *   w0      [d_out, d_in]  frozen base weight (nn.Linear layout), dtype
 *   lora_a  [rank, d_in]   adapter down-projection, dtype
 *   lora_b  [d_out, rank]  adapter up-projection, dtype
 *   row_gate[M] float32    per-row gate; NULL means all zeros (base layer only)
 *   scale                  adapter scale (alpha / r under the standard LoRA reading)
 *   y       [M, d_out]     output, dtype; must not overlap any input
 *
 * Arithmetic: bf16 tensor-core products with fp32 accumulation. The adapter's
 * intermediate T = scale * g * (X A^T) is accumulated in fp32 and rounded once to bf16
 * before the up-projection, which accumulates into the same fp32 accumulator as X W0^T;
 * Y is rounded once to the output dtype. With dtype UNO_F32 the inputs are rounded to
 * bf16 (round-to-nearest-even) on the device first and Y is written as float32.
 *
 * Limits (else UNO_ERR_UNSUPPORTED): d_in and d_out multiples of 64; rank a multiple of 8
 * with 8 <= rank <= 256; 1 <= M <= 2^20; d_in, d_out <= 65536.
 * Workspace: uno_gated_lora_linear_workspace_size(M, d_in, d_out, rank, dtype) bytes.
 * ====================================================================================== */
size_t uno_gated_lora_linear_workspace_size(int64_t M, int64_t d_in, int64_t d_out,
                                            int64_t rank, uno_dtype dtype);

uno_status uno_gated_lora_linear(const void* x, const void* w0, const void* lora_a,
                                 const void* lora_b, const float* row_gate, float scale,
                                 int64_t M, int64_t d_in, int64_t d_out, int64_t rank,
                                 uno_dtype dtype, void* y, void* workspace,
                                 size_t workspace_bytes, uno_stream_t stream);

/* ======================================================================================
 * Lossless block verify
 *
 * For each sequence b of a batch, a block of K positions was drafted in one forward.
 * verifier_logits[b, i] gives the verifier's (frozen base model's) next-token logits at
 * block position i, drafter_logits[b, i] the drafter's (model + gated LoRA). Both rows
 * are warped the same way: z = logit / temperature; top-k (exactly k kept, ties to the
 * lower token id); softmax; top-p (shortest prefix of the (probability desc, id asc)
 * order whose cumulative mass is >= top_p, the crossing token included); renormalise.
 * Call the results p_i and q_i.
 *
 *   x_0 = pos0_tokens[b] if given and >= 0, else the inverse-CDF draw of p_0 with
 *         uniforms[b,0,0]
 *   d_i = draft_tokens[b,i], or the inverse-CDF draw of q_i with uniforms[b,i,0], i >= 1
 *   draft i is accepted iff uniforms[b,i,1] * q_i(d_i) < p_i(d_i)  (prob. min(1, p/q))
 *   n = 1 + number of leading accepted drafts (position 0 is always emitted)
 *   at the first rejection j: next = inverse-CDF draw of normalise(max(0, p_j - q_j))
 *   with uniforms[b,j,2] (p_j itself if that has no mass); next = -1 if all accepted.
 *
 * The inverse-CDF draw of a distribution w with uniform u returns the smallest token id t
 * (ascending) whose cumulative mass sum_{s<=t} w_s exceeds u * sum(w).
 * The acceptance probability is 1 - TV(p_i, q_i) and every emitted token is distributed
 * as p_i: the verify is lossless. Source: LoopUno project page, "How it works" (the
 * unmodified model verifies the block and keeps the longest correct prefix; the first
 * position is always the exact AR token) and "Training is self-distillation" (acceptance
 * probability is exactly 1 - TV); uno-qwen3-8B model card, "Evaluation protocol"
 * (temperature 1.0, top-p 0.95, top-k 50, block 16).
 *
 *   verifier_logits [B, K, V]  dtype (bf16 or f32); all K rows used
 *   drafter_logits  [B, K, V]  dtype; rows i >= 1 used (row 0 is never read)
 *   temperature     > 0
 *   top_k           0 = off; else 1 <= top_k <= 1024 (top_k >= V is the same as off)
 *   top_p           (0, 1) filters; >= 1 = off
 *   draft_tokens    [B, K] int32 or NULL (column 0 ignored); NULL: drawn from q_i
 *   pos0_tokens     [B] int32 or NULL; NULL or an entry < 0: drawn from p_0 (so a
 *                   previous step's out_next_token can be passed as is: -1 when all of
 *                   its drafts were accepted)
 *   uniforms        [B, K, 3] float32 in [0, 1): (sample, accept, resample)
 *   out_tokens      [B, K] int32: x_0, d_1 .. d_{n-1}, then -1
 *   out_count       [B] int32: n
 *   out_next_token  [B] int32 or NULL: the correction token, -1 if every draft was accepted
 *   out_p_tok       [B, K] float32 or NULL: p_i(token_i) (token_0 = x_0, token_i = d_i)
 *   out_q_tok       [B, K] float32 or NULL: q_i(d_i); 0 at i = 0
 *   out_tv          [B, K] float32 or NULL: TV(p_i, q_i) for i >= 1, 0 at i = 0
 *
 * Logits must be finite. Limits (else UNO_ERR_UNSUPPORTED): 1 <= K <= 32, 1 <= V < 2^31,
 * B >= 0 (B = 0 does nothing), B * K * V < 2^40.
 * Workspace: uno_block_verify_workspace_size(B, K, V, top_k, top_p, dtype) bytes, the size
 * the fastest path uses. With top_k off and bf16 logits that includes each row's candidate
 * list (every token whose logit is near enough to the row's largest to be in the nucleus,
 * 128 KiB per row); a workspace of at least uno_block_verify_min_workspace_size(...) bytes
 * is also accepted, and the call then weighs every item from the logits instead (slower,
 * same results). The two sizes are equal when top_k is on.
 * ====================================================================================== */
size_t uno_block_verify_workspace_size(int32_t B, int32_t K, int32_t V, int32_t top_k,
                                       float top_p, uno_dtype dtype);
size_t uno_block_verify_min_workspace_size(int32_t B, int32_t K, int32_t V, int32_t top_k,
                                           float top_p, uno_dtype dtype);

uno_status uno_block_verify(const void* verifier_logits, const void* drafter_logits,
                            uno_dtype dtype, int32_t B, int32_t K, int32_t V,
                            float temperature, int32_t top_k, float top_p,
                            const int32_t* draft_tokens, const int32_t* pos0_tokens,
                            const float* uniforms, int32_t* out_tokens, int32_t* out_count,
                            int32_t* out_next_token, float* out_p_tok, float* out_q_tok,
                            float* out_tv, void* workspace, size_t workspace_bytes,
                            uno_stream_t stream);

/* ======================================================================================
 * Block verify without a caller-supplied workspace
 *
 * The Uno pages have no counterpart to this call: it is a convenience of this library.
 * It takes the arguments of uno_block_verify except the workspace and gives the same
 * results. It serves callers that cannot allocate device memory where they call the
 * verify: a plugin or embedded runtime that receives device pointers and a stream from
 * its host application but has no allocator of its own, or a latency-bound serving loop
 * that may not call cudaMalloc (which can synchronise the whole device).
 *
 * Its scratch is a fixed array of UNO_NOALLOC_SCRATCH_BYTES compiled into the library; every
 * device that loads the library holds it until the process exits. The call allocates and
 * frees nothing. The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture. All calls on a device
 * share the array, which keeps the last call's contents (nothing in it needs to start at
 * zero); calls that can overlap on the GPU race on it, so order them on one stream or
 * synchronise between them.
 *
 * It uses the candidate lists when the array holds them, and otherwise the smaller workspace.
 * Errors: as uno_block_verify, plus UNO_ERR_UNSUPPORTED when the batch needs more scratch
 * than the array holds (uno_block_verify_min_workspace_size(...) > UNO_NOALLOC_SCRATCH_BYTES;
 * the 64 x 16 x 151936 top-k 50 batch needs about 9.4 MiB).
 * ====================================================================================== */
#define UNO_NOALLOC_SCRATCH_BYTES (16u << 20)

uno_status uno_block_verify_noalloc(const void* verifier_logits, const void* drafter_logits,
                                    uno_dtype dtype, int32_t B, int32_t K, int32_t V,
                                    float temperature, int32_t top_k, float top_p,
                                    const int32_t* draft_tokens, const int32_t* pos0_tokens,
                                    const float* uniforms, int32_t* out_tokens,
                                    int32_t* out_count, int32_t* out_next_token,
                                    float* out_p_tok, float* out_q_tok, float* out_tv,
                                    uno_stream_t stream);

/* ======================================================================================
 * Block noising, noise mode random_uniform
 *
 * The block-noised copy that the student (training) and the drafter (decode) read: in
 * every block, position 0 keeps its token and each draft position i = 1..K-1 gets a token
 * drawn uniformly from the vocabulary by the supplied uniform:
 *   noised[b, 0] = clean[b, 0]
 *   noised[b, i] = min(V - 1, floor(uniforms[b, i] * V))          (i >= 1, fp64, exact)
 *   row_gate[b * K + i] = 0 at i = 0, 1 at i >= 1  (the adapter's gate for these rows)
 * Source: LoopUno project page, "Training is self-distillation" (the student is the model
 * with its LoRA on a block-noised copy of each sequence) and "How it works" (position 0 is
 * the exact AR token; the adapter is on only for noise positions); uno-qwen3-8B model
 * card, "Evaluation protocol" (noise mode random_uniform).
 *
 *   clean_tokens  [B, K] int32
 *   uniforms      [B, K] float32 in [0, 1) (uniforms[b, 0] is not read; 1.0 maps to V - 1)
 *   noised_tokens [B, K] int32; may be clean_tokens itself (each output element depends
 *                 only on the same input element)
 *   row_gate      [B * K] float32 or NULL
 *
 * Device pointers, 4-byte aligned. Limits (else UNO_ERR_INVALID_ARG): B >= 0, K >= 1,
 * 1 <= V < 2^24. B = 0 launches nothing. No workspace.
 * ====================================================================================== */
uno_status uno_block_noise(const int32_t* clean_tokens, const float* uniforms, int32_t B, int32_t K,
                           int32_t V, int32_t* noised_tokens, float* row_gate, uno_stream_t stream);

/* ======================================================================================
 * TV self-distillation loss and its gradient
 *
 *   p_t = softmax(teacher_logits[t]), q_t = softmax(student_logits[t])   (T = 1, no filter)
 *   tv[t] = 1/2 sum_v |p_t,v - q_t,v|
 *   mean  = sum over masked tokens of tv[t] / N_mask        (0 when no token is masked in)
 *   grad_student[t, v] = grad_scale / N_mask * q_t,v * (s_v - sum_w q_t,w s_w)
 *                        with s = 1/2 sign(q_t - p_t), sign(0) = 0; 0 on unmasked tokens
 *
 * The teacher (frozen model on the clean copy) is constant; the student is model + LoRA
 * on the block-noised copy. Source: LoopUno project page, "Training is
 * self-distillation" (TV distance between the two next-token distributions on the
 * response tokens) and "Setup / Recipe" (objective: TV distance to the frozen model's own
 * distribution).
 *
 *   teacher_logits, student_logits [N, V] dtype (bf16 or f32)
 *   response_mask  [N] uint8 or NULL (NULL: every token counts)
 *   grad_scale     dL/dmean (1 for the plain mean)
 *   out_tv         [N] float32
 *   out_mean       [1] float32
 *   grad_student   [N, V] dtype or NULL (NULL: loss only)
 *
 * Logits must be finite. Limits (else UNO_ERR_UNSUPPORTED): 1 <= V < 2^31, N >= 0,
 * N * V < 2^40.
 * Workspace: uno_tv_loss_workspace_size(N, V, dtype) bytes.
 * ====================================================================================== */
size_t uno_tv_loss_workspace_size(int64_t N, int64_t V, uno_dtype dtype);

uno_status uno_tv_loss(const void* teacher_logits, const void* student_logits,
                       uno_dtype dtype, int64_t N, int64_t V, const uint8_t* response_mask,
                       float grad_scale, float* out_tv, float* out_mean, void* grad_student,
                       void* workspace, size_t workspace_bytes, uno_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* UNO_H */

/*
 * dd.h -- C ABI of libdd: one denoising step of block discrete-diffusion
 * decoding on an NVIDIA B200 (sm_100a).
 *
 * What the step computes ("DiffusionGemma Technical Report", paperfeed
 * review, section "The mechanism: an AR model turned inside out"):
 *   - a 256-token canvas whose queries attend bidirectionally to the whole
 *     canvas and to a causally encoded prefix KV cache;
 *   - a sampler that turns each position's temperature-scaled logits into a
 *     new token, a confidence and an entropy, then re-corrupts positions to
 *     uniformly random vocabulary tokens (multinomial noise, not [MASK]);
 *   - about 12 such passes per 256-token block.
 *
 * Conventions for every entry point:
 *   - Ownership: the caller owns every buffer.  libdd never allocates device
 *     or pinned memory; scratch space is the caller's `workspace`.
 *   - Pointers are DEVICE pointers unless the name ends in `_host`.
 *   - Tensors are dense row-major ("C order"), last dimension fastest, with
 *     the shapes given below.  Device pointers must be 16-byte aligned.
 *   - Every call is asynchronous on `stream` (0 = the legacy default stream)
 *     and makes no host synchronisation, except dd_query_device_error and
 *     dd_denoise_block_adaptive (which reads the halt flags after every
 *     step; dd_denoise_block_adaptive_graph_* keep that loop on the device).
 *   - Errors: arguments are validated on the host BEFORE any launch.  Invalid
 *     shapes/pointers return DD_ERR_INVALID_ARG, shapes without a kernel
 *     return DD_ERR_UNSUPPORTED, a too-small workspace DD_ERR_WORKSPACE, a
 *     failed launch DD_ERR_CUDA.  dd_last_error() then holds a message
 *     (thread-local).  Nothing aborts or throws across this boundary.
 *   - Device-side faults that kernels detect themselves (a pipeline wait that
 *     exceeded its time limit) are latched in the first 16 bytes of the
 *     workspace and read back by dd_query_device_error.
 *   - A workspace must be cleared once with dd_workspace_init before its
 *     first use.  The sampler keeps a small state in it (a work counter and
 *     per-row maxima) and per-chunk records, all of which every completed
 *     call leaves cleared, so sampler calls of any shape may share a
 *     workspace.  The attention path keeps a pair of counters per (batch
 *     row, kv head, query-tile pair) at the start of its scratch (split
 *     partials done, merge CTAs that have seen them), which every completed
 *     call also leaves cleared; its split partials are not cleared and are
 *     laid out for one geometry.  So a dd_denoise_block or
 *     dd_denoise_block_adaptive workspace serves one geometry (batch,
 *     canvas, heads, prefix lengths, vocabulary); clear it with
 *     dd_workspace_init before using it for another.  After a call that
 *     failed on the device, clear the workspace again.
 *   - There is no CPU fallback: if the CUDA kernels cannot run, calls fail.
 */
#ifndef DD_H_
#define DD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DD_API __attribute__((visibility("default")))
#else
#define DD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dd_stream_t; /* == cudaStream_t */

typedef enum {
  DD_OK = 0,
  DD_ERR_INVALID_ARG = 1,
  DD_ERR_UNSUPPORTED = 2,
  DD_ERR_WORKSPACE = 3,
  DD_ERR_CUDA = 4,
  DD_ERR_DEVICE_TIMEOUT = 5,
  DD_ERR_DEVICE_BOUNDS = 6
} dd_status;

/* Element types.  DD_E4M3 (8-bit floating point, OCP OFP8 E4M3 encoding:
 * bias 7, 3 mantissa bits, largest finite value 448) is taken only by
 * dd_canvas_attn_fp8, with one scale factor per tensor. */
typedef enum { DD_BF16 = 0, DD_F32 = 1, DD_E4M3 = 2 } dd_dtype;

/* Geometry of one canvas-attention call.
 *   batch     B >= 1 canvases (batch rows)
 *   canvas    C >= 1 positions per canvas (256 in the method)
 *   heads_q   Hq query heads; heads_kv Hkv kv heads, Hq % Hkv == 0.  Query
 *             head h reads kv head h / (Hq / Hkv) (grouped-query attention;
 *             the pages do not state the head mapping, this is the usual one).
 *   head_dim  D in {64, 128}
 *   scale     softmax scale (1/sqrt(D) in every workload here)
 *   dtype     DD_BF16 (tensor cores, fp32 accumulation), DD_F32 (fp32 FMA)
 *             or DD_E4M3 (tensor cores, fp32 accumulation; dd_canvas_attn_fp8) */
typedef struct {
  int batch, canvas, heads_q, heads_kv, head_dim;
  float scale;
  dd_dtype dtype;
} dd_attn_desc;

/* Workspace bytes that dd_canvas_attn (or dd_canvas_attn_fp8, for a
 * DD_E4M3 desc) needs for this geometry and these prefix lengths
 * (cu_prefix_host: [B+1] host array, see dd_canvas_attn).
 * Returns 0 if the arguments are invalid. */
DD_API size_t dd_canvas_attn_workspace(const dd_attn_desc* desc, const int32_t* cu_prefix_host);

/* Bidirectional canvas attention over [prefix KV || canvas KV]
 * ("DiffusionGemma Technical Report", "The mechanism": the canvas is refined
 * with full bidirectional attention inside the canvas while attending to the
 * causally encoded cache).  For batch row b, position i, query head h with
 * g = h / (Hq/Hkv), the keys are the L_b prefix rows of b followed by the C
 * canvas rows of b, all unmasked, under ONE softmax:
 *   O[b,i,h,:] = sum_j softmax_j(scale * <q, k_j>) v_j
 * Arguments (element type = desc->dtype):
 *   q            [B, C, Hq, D]
 *   k_canvas     [B, C, Hkv, D]     v_canvas  same
 *   k_prefix     [sum_b L_b, Hkv, D] packed; rows cu_prefix[b]..cu_prefix[b+1]-1
 *   v_prefix     same
 *   cu_prefix    device int32 [B+1], cu_prefix[0] = 0, non-decreasing;
 *                L_b = cu_prefix[b+1] - cu_prefix[b] may be 0
 *   cu_prefix_host  host copy of the same values.  It plans the launch and,
 *                for batches of up to 128 rows, carries each row's prefix
 *                offset into the kernels, which then address the prefix
 *                with it; wider batches read cu_prefix on the device.  The
 *                two must agree, which is not checked (reads stay inside
 *                the prefix tensor, whose extent is cu_prefix_host[B])
 *   out          [B, C, Hq, D], element type = desc->dtype
 *   lse          optional fp32 [B, Hq, C]: natural-log sum of exp of scores
 *   workspace    >= dd_canvas_attn_workspace(...) bytes, 256-byte aligned
 * desc->dtype DD_E4M3 is rejected here (DD_ERR_INVALID_ARG): the 8-bit path
 * is dd_canvas_attn_fp8. */
DD_API dd_status dd_canvas_attn(const dd_attn_desc* desc, const void* q, const void* k_canvas,
                         const void* v_canvas, const void* k_prefix, const void* v_prefix,
                         const int32_t* cu_prefix, const int32_t* cu_prefix_host, void* out,
                         float* lse, void* workspace, size_t workspace_bytes, dd_stream_t stream);

/* Per-tensor scale factors of 8-bit attention inputs: the value of an
 * element is its E4M3 value times its tensor's factor.  `k` covers both
 * k_prefix and k_canvas, `v` both v_prefix and v_canvas.  Finite and > 0. */
typedef struct {
  float q, k, v;
} dd_fp8_scales;

/* dd_canvas_attn on 8-bit inputs: the same definition and layouts, with
 * desc->dtype = DD_E4M3, q / k_* / v_* holding E4M3 bytes (one byte per
 * element) and `scales` their factors:
 *   O[b,i,h,:] = f_v * sum_j softmax_j(scale * f_q * f_k * <q, k_j>) v_j
 * The pages quote their step times for 8-bit inference ("DiffusionGemma
 * Technical Report", "The numbers, honestly"); this is the attention of
 * that step on the tensor cores' 8-bit path (kind::f8f6f4, fp32
 * accumulation).  The softmax probabilities are rounded to E4M3 for the
 * P.V product (relative rounding error <= 2^-4 per probability); the
 * row sums and the output use the unrounded fp32 values.
 *   out   [B, C, Hq, D] bf16
 *   lse   optional fp32 [B, Hq, C]
 * Requires head_dim 128 and (heads_q / heads_kv) dividing 128, else
 * DD_ERR_UNSUPPORTED.  Same workspace as dd_canvas_attn
 * (dd_canvas_attn_workspace with the DD_E4M3 desc). */
DD_API dd_status dd_canvas_attn_fp8(const dd_attn_desc* desc, const void* q,
                                    const void* k_canvas, const void* v_canvas,
                                    const void* k_prefix, const void* v_prefix,
                                    const int32_t* cu_prefix, const int32_t* cu_prefix_host,
                                    const dd_fp8_scales* scales, void* out, float* lse,
                                    void* workspace, size_t workspace_bytes, dd_stream_t stream);

/* Sampler parameters for one step.
 *   temperature   tau > 0; logits are divided by it (the method anneals it
 *                 0.8 -> 0.4 over the steps; the caller passes each step's)
 *   renoise_rate  probability in [0,1] that a position is re-noised
 *   seed          Philox4x32-10 key
 *   step          Philox counter word 2 (the denoising step)
 *   row_offset    global index of row 0 of this call (Philox counter word 1
 *                 is row_offset + local row), so that a batch split across
 *                 calls draws the same numbers as one call. */
typedef struct {
  float temperature;
  float renoise_rate;
  uint64_t seed;
  uint32_t step;
  uint32_t row_offset;
} dd_sample_params;

/* Workspace bytes that dd_sample_renoise needs (0 on invalid arguments). */
DD_API size_t dd_sample_renoise_workspace(int rows, int vocab, dd_dtype dtype);

/* One sampler + re-noise step over `rows` positions ("DiffusionGemma
 * Technical Report", "The mechanism": temperature-scaled logits give
 * per-position entropies; positions not kept are re-noised to uniformly
 * random vocabulary tokens; "Training": each token is corrupted
 * independently with a probability).  For global row r and vocab index v,
 * with z = logit / tau and Philox4x32-10 words x(stream, v) under key = seed,
 * counter (v >> 2, r, step, stream), word v & 3:
 *   pred      = argmax_v z_v - ln(-ln U(x(0, v))),  U(x) = (2 (x >> 9) + 1) 2^-24
 *               (Gumbel-max: a draw from softmax(z); lowest v on exact ties)
 *   conf      = softmax(z)[pred]
 *   entropy   = -sum_v p_v ln p_v, p = softmax(z)
 *   renoised  = U(x(1, 0)) < renoise_rate   (fp32 compare)
 *   token     = renoised ? (x(2, 0) * V) >> 32 : pred
 * Arguments:
 *   logits       [rows, V] of `dtype` with `row_stride` elements between rows
 *                (row_stride >= V)
 *   tokens_out   int32 [rows] (required)
 *   pred_out     int32 [rows] or NULL
 *   conf_out     fp32 [rows] (required)
 *   entropy_out  fp32 [rows] or NULL
 *   renoised_out uint8 [rows] or NULL
 *   workspace    >= dd_sample_renoise_workspace(rows, V, dtype) bytes */
DD_API dd_status dd_sample_renoise(const void* logits, dd_dtype dtype, int rows, int vocab,
                            int64_t row_stride, const dd_sample_params* params,
                            int32_t* tokens_out, int32_t* pred_out, float* conf_out,
                            float* entropy_out, uint8_t* renoised_out, void* workspace,
                            size_t workspace_bytes, dd_stream_t stream);

/* Canvas initialisation to uniformly random vocabulary tokens ("The
 * mechanism": a canvas of noise): canvas[r] = (x * V) >> 32 with x the word
 * for key = seed, counter (0, row_offset + r, 0, 3), word 0.
 *   canvas  int32 [rows] */
DD_API dd_status dd_init_canvas(int32_t* canvas, int rows, int vocab, uint64_t seed, uint32_t row_offset,
                         dd_stream_t stream);

/* Workspace bytes for dd_denoise_block, or for dd_denoise_block_fp8 when
 * desc->dtype is DD_E4M3 (the larger of the two steps' needs). */
DD_API size_t dd_denoise_block_workspace(const dd_attn_desc* desc, const int32_t* cu_prefix_host,
                                  int vocab);

/* The inner loop of one block: `steps` denoising passes ("about 12 forward
 * passes per 256-token block", "The mechanism").  Step s (0-based) runs
 * dd_canvas_attn on the step's canvas Q/K/V and dd_sample_renoise on the
 * step's logits with Philox step = step0 + s, temperature_host[s] and
 * rate_host[s]; the canvas after step s is its tokens.  Steps are
 * independent of the previous canvas (the model that would map the canvas
 * to Q/K/V and logits is outside this library), so restarting at step0 = k
 * reproduces steps k.. exactly.
 * Arguments (R = B*C rows, element type = desc->dtype):
 *   q_steps        [S, B, C, Hq, D];  kc_steps, vc_steps [S, B, C, Hkv, D]
 *   k_prefix, v_prefix, cu_prefix, cu_prefix_host: as dd_canvas_attn
 *   attn_out       [S, B, C, Hq, D]
 *   logits_steps   [S, R, V] (dtype as desc->dtype)
 *   rate_host, temperature_host   host fp32 [S]
 *   canvas         int32 [R]: the canvas after the last step
 *   canvas_history int32 [S, R] or NULL: every step's canvas
 *   conf_steps     fp32 [S, R] or NULL: every step's confidences
 *   workspace      >= dd_denoise_block_workspace(...) bytes */
DD_API dd_status dd_denoise_block(const dd_attn_desc* desc, int steps, const void* q_steps,
                           const void* kc_steps, const void* vc_steps, const void* k_prefix,
                           const void* v_prefix, const int32_t* cu_prefix,
                           const int32_t* cu_prefix_host, void* attn_out,
                           const void* logits_steps, int vocab, const float* rate_host,
                           const float* temperature_host, uint64_t seed, uint32_t step0,
                           int32_t* canvas, int32_t* canvas_history, float* conf_steps,
                           void* workspace, size_t workspace_bytes, dd_stream_t stream);

/* dd_denoise_block with 8-bit attention inputs: step s runs
 * dd_canvas_attn_fp8 with the factors scales_host[s], then
 * dd_sample_renoise on bf16 logits.  desc->dtype must be DD_E4M3; q_steps,
 * kc_steps, vc_steps, k_prefix and v_prefix are E4M3 with the shapes of
 * dd_denoise_block; attn_out is bf16 [S, B, C, Hq, D]; logits_steps is bf16
 * [S, R, V].  scales_host: host array of `steps` factor sets, each
 * validated like dd_canvas_attn_fp8's (DD_ERR_INVALID_ARG names the step).
 * Every other argument, the workspace query and the results' meaning are
 * those of dd_denoise_block. */
DD_API dd_status dd_denoise_block_fp8(const dd_attn_desc* desc, int steps, const void* q_steps,
                               const void* kc_steps, const void* vc_steps, const void* k_prefix,
                               const void* v_prefix, const int32_t* cu_prefix,
                               const int32_t* cu_prefix_host, const dd_fp8_scales* scales_host,
                               void* attn_out, const void* logits_steps, int vocab,
                               const float* rate_host, const float* temperature_host,
                               uint64_t seed, uint32_t step0, int32_t* canvas,
                               int32_t* canvas_history, float* conf_steps, void* workspace,
                               size_t workspace_bytes, dd_stream_t stream);

/* A block loop captured once and replayed with a single launch.  The loop
 * takes 4 kernels per step (attention, split combine, sampler pass, row
 * merge).  At about 0.1 ms per step, launching them one by one from the
 * host shows up in the block time, and a graph removes that cost.
 *   dd_denoise_block_graph_create captures one dd_denoise_block call with
 *     exactly these arguments (the same as dd_denoise_block, without the
 *     stream) into a CUDA graph and instantiates it.  It validates the
 *     arguments like dd_denoise_block, launches nothing, and on success
 *     stores a handle in *out (NULL on failure).  The handle is a small host
 *     object; no device memory is allocated.
 *   dd_denoise_block_graph_launch replays the captured call on `stream`:
 *     the same pointers, sizes, rates, temperatures, seed and step0.  New
 *     inputs enter by overwriting the contents of the captured buffers.
 *     Every buffer must stay allocated while the handle exists.  Replays
 *     that may overlap in time must not share a workspace.
 *   dd_denoise_block_graph_destroy frees the handle (NULL is accepted).
 * A replay gives results identical to the eager call. */
typedef struct dd_block_graph_st* dd_block_graph;
DD_API dd_status dd_denoise_block_graph_create(
    dd_block_graph* out, const dd_attn_desc* desc, int steps, const void* q_steps,
    const void* kc_steps, const void* vc_steps, const void* k_prefix, const void* v_prefix,
    const int32_t* cu_prefix, const int32_t* cu_prefix_host, void* attn_out,
    const void* logits_steps, int vocab, const float* rate_host, const float* temperature_host,
    uint64_t seed, uint32_t step0, int32_t* canvas, int32_t* canvas_history, float* conf_steps,
    void* workspace, size_t workspace_bytes);
DD_API dd_status dd_denoise_block_graph_launch(dd_block_graph graph, dd_stream_t stream);
DD_API dd_status dd_denoise_block_graph_destroy(dd_block_graph graph);

/* Self-conditioning soft embedding ("DiffusionGemma Technical Report",
 * "The mechanism", self-conditioning paragraph: the previous step's
 * predicted token distribution, pushed through the embedding matrix E, is
 * the input of a small MLP that conditions the next step).  This computes
 * the contraction; dd_ffw is the MLP that follows it, and
 * dd_self_condition runs both:
 *   out[r, :] = sum_v softmax(logits[r, :] / temperature)_v * E[v, :]
 * Arguments:
 *   logits       bf16 [rows, vocab] with row_stride elements between rows
 *                (row_stride >= vocab, a multiple of 8)
 *   dtype        DD_BF16 (the only type taken; others DD_ERR_UNSUPPORTED)
 *   temperature  tau >= 1e-3 (the distribution the sampler draws from)
 *   emb          E, bf16 [vocab, d], row-major; d a multiple of 64
 *                (else DD_ERR_UNSUPPORTED)
 *   out          bf16 [rows, d]
 *   workspace    >= dd_soft_embed_workspace(rows, vocab, d) bytes, 256-byte
 *                aligned (row log-sum-exps and fp32 partial sums)
 * The probabilities are rounded to bf16 for the tensor-core product
 * (relative error <= 2^-8 each); accumulation is fp32; the partial sums
 * of the vocabulary splits are added in a fixed order (the result does not
 * depend on scheduling).  Returns 0 from the workspace query on invalid
 * arguments. */
DD_API size_t dd_soft_embed_workspace(int rows, int vocab, int d);
DD_API dd_status dd_soft_embed(const void* logits, dd_dtype dtype, int rows, int vocab,
                               int64_t row_stride, float temperature, const void* emb, int d,
                               void* out, void* workspace, size_t workspace_bytes,
                               dd_stream_t stream);

/* Self-conditioning MLP ("DiffusionGemma Technical Report", "The mechanism",
 * self-conditioning paragraph: the soft embedding u = p0 E goes through "a
 * small MLP (7.8M parameters)", z_t = FFW(u)).  The pages give only the
 * size; the MLP is read as two dense layers with a GELU between them:
 *   hid[r, :] = GELU(u[r, :] W1 + b1),   GELU(x) = x Phi(x) (erf form)
 *   out[r, :] = hid[r, :] W2 + b2
 * At d = 2048 and hidden = 1904 that is 7,802,784 parameters.  Both layers
 * run on the tensor cores (bf16 operands, fp32 accumulation); the hidden
 * activations and the output are rounded to bf16 (relative error <= 2^-8
 * each).
 *   u        bf16 [rows, d]
 *   w1       bf16 [d, hidden], row-major;  b1 bf16 [hidden]
 *   w2       bf16 [hidden, d], row-major;  b2 bf16 [d]
 *   out      bf16 [rows, d]
 *   workspace >= dd_ffw_workspace(rows, d, hidden) bytes, 256-byte aligned
 *            (error word and the bf16 hidden activations)
 * d and hidden must be multiples of 16 (>= 16), else DD_ERR_UNSUPPORTED
 * (DD_ERR_INVALID_ARG below 16).  dd_ffw_workspace returns 0 on invalid
 * shapes. */
DD_API size_t dd_ffw_workspace(int rows, int d, int hidden);
DD_API dd_status dd_ffw(const void* u, int rows, int d, int hidden, const void* w1,
                        const void* b1, const void* w2, const void* b2, void* out,
                        void* workspace, size_t workspace_bytes, dd_stream_t stream);

/* The whole self-conditioning signal of a step: dd_soft_embed of the
 * logits, then dd_ffw,  out = FFW(softmax(logits / temperature) E).
 * Arguments as dd_soft_embed (logits, dtype, rows, vocab, row_stride,
 * temperature, emb, d; d a multiple of 64) and dd_ffw (w1, b1, hidden, w2,
 * b2, out).  u_out: bf16 [rows, d] receiving the soft embedding, or NULL
 * (it then lives in the workspace).  Every argument is checked before the
 * first launch.  workspace >= dd_self_condition_workspace(rows, vocab, d,
 * hidden) bytes, 256-byte aligned; 0 on invalid shapes. */
DD_API size_t dd_self_condition_workspace(int rows, int vocab, int d, int hidden);
DD_API dd_status dd_self_condition(const void* logits, dd_dtype dtype, int rows, int vocab,
                                   int64_t row_stride, float temperature, const void* emb, int d,
                                   const void* w1, const void* b1, int hidden, const void* w2,
                                   const void* b2, void* out, void* u_out, void* workspace,
                                   size_t workspace_bytes, dd_stream_t stream);

/* dd_sample_renoise without a workspace, for callers that may not allocate
 * device memory (code inside another framework's memory pool or fixed
 * budget, plugin or callback code handed only its input and output
 * pointers, latency-critical loops that cannot accept cudaMalloc's device
 * synchronisation).  The paper has no counterpart: this is a deployment
 * variant of the same sampler step.
 * Arguments and results: exactly as dd_sample_renoise, minus the workspace.
 * Scratch: a static device array of 4 MiB that the library holds on every
 * GPU it is loaded on until the process exits.  A call needs
 * dd_sample_renoise_workspace(rows, vocab, dtype) bytes of it (about 512
 * bytes, plus 128 bytes per row, plus 16 bytes per 2048 vocabulary entries
 * per row: up to 1927 rows at V = 262144); larger calls return
 * DD_ERR_UNSUPPORTED before touching the GPU.  The function allocates
 * nothing: no cudaMalloc, cudaFree or allocating library call.
 * Arguments are checked before any GPU work is queued (a rejected call
 * queues nothing); rows == 0 returns DD_OK after the same checks as
 * dd_sample_renoise.  Each call clears, on the stream and before its
 * kernels, the part of the array it reads before writing (an error word, a
 * work counter and its rows' maxima, about 512 + 128 * rows bytes), so a
 * call that failed on the device does not affect later calls.
 * The first call in each CUDA context (on each device, and again after a
 * device reset) looks up the array's device address with
 * cudaGetSymbolAddress, so make that call before any stream capture.
 * Every call shares the array: calls that overlap on the GPU (two streams,
 * or two host threads) race and may return wrong results.  A bounds error
 * that the merge kernel detects is cleared by the next call and is not
 * reported by this entry point (dd_sample_renoise with
 * dd_query_device_error reports it). */
DD_API dd_status dd_sample_renoise_noalloc(const void* logits, dd_dtype dtype, int rows, int vocab,
                                           int64_t row_stride, const dd_sample_params* params,
                                           int32_t* tokens_out, int32_t* pred_out,
                                           float* conf_out, float* entropy_out,
                                           uint8_t* renoised_out, dd_stream_t stream);

/* ---- The pages' own sampler policy ("DiffusionGemma Technical Report",
 * "The mechanism", sampler paragraph): temperature annealed 0.8 -> 0.4,
 * positions accepted greedily from lowest to highest entropy until a
 * cumulative entropy budget (b = 0.1) is exhausted and the rest re-noised to
 * uniform random tokens, early halt when the mean canvas entropy is below
 * 0.005 and the prediction is stable across two steps.  The scheduled-rate
 * loop (dd_denoise_block) stays the default; these calls are the pages'
 * alternative. */

/* Entropy-budget acceptance for `batch` canvases of `canvas` positions
 * (rows b*canvas .. b*canvas+canvas-1): positions are taken in increasing
 * entropy (equal entropies: lower position first) and accepted while the
 * float64 running sum of accepted entropies stays <= budget; the first that
 * would exceed it ends the acceptance.  tokens_out = pred at accepted
 * positions, elsewhere the uniform replacement token of the row as in
 * dd_sample_renoise: (x(2, 0) * V) >> 32 under key seed, counter
 * (0, row_offset + row, step, 2).
 *   entropy      fp32 [rows] (as dd_sample_renoise outputs it)
 *   pred         int32 [rows]
 *   tokens_out   int32 [rows]
 *   accepted_out uint8 [rows] or NULL
 * canvas must be 1..1024. */
DD_API dd_status dd_entropy_accept(const float* entropy, const int32_t* pred, int batch, int canvas,
                                   int vocab, float budget, uint64_t seed, uint32_t step,
                                   uint32_t row_offset, int32_t* tokens_out, uint8_t* accepted_out,
                                   dd_stream_t stream);

/* Early-halt test, per canvas: a canvas not yet done halts at this step when
 * the float64 mean of its entropies (summed in position order) is below
 * `threshold` and pred equals pred_prev at every position (pred_prev NULL:
 * no previous step, no halt).  Halting sets done[b] = 1 and halt_step[b] =
 * step; canvases already done are left alone.
 *   entropy fp32 [rows]; pred, pred_prev int32 [rows]
 *   done uint8 [batch] (in/out); halt_step int32 [batch] (out) */
DD_API dd_status dd_stop_check(const float* entropy, const int32_t* pred, const int32_t* pred_prev,
                               int batch, int canvas, float threshold, int32_t step, uint8_t* done,
                               int32_t* halt_step, dd_stream_t stream);

/* Workspace bytes for dd_denoise_block_adaptive. */
DD_API size_t dd_denoise_block_adaptive_workspace(const dd_attn_desc* desc,
                                                  const int32_t* cu_prefix_host, int vocab);

/* The block loop under the pages' policy: up to max_steps steps; step s runs
 * dd_canvas_attn and the sampler (temperature_host[s], Philox step
 * step0 + s, no scheduled re-noise), then dd_stop_check against step s - 1's
 * predictions, then dd_entropy_accept into `canvas`.  A canvas that halts at
 * step s takes its whole prediction as its final canvas and is left
 * unchanged by later steps; the loop ends when every canvas has halted or
 * after max_steps.  Unlike every other call here, it synchronises `stream`
 * once per step to read the halt flags (that is what lets it stop early).
 * Arguments as dd_denoise_block, plus:
 *   temperature_host  host fp32 [max_steps] (the pages anneal 0.8 -> 0.4)
 *   budget, stop_entropy  the pages' b = 0.1 and 0.005
 *   canvas            int32 [R], in/out (its initial content is only the
 *                     model's input, which is synthetic here)
 *   canvas_history    int32 [max_steps, R] or NULL: the canvas after each
 *                     step run
 *   halt_step         device int32 [B]: the step each canvas halted at, or -1
 *   steps_run         host int: steps run */
DD_API dd_status dd_denoise_block_adaptive(
    const dd_attn_desc* desc, int max_steps, const void* q_steps, const void* kc_steps,
    const void* vc_steps, const void* k_prefix, const void* v_prefix, const int32_t* cu_prefix,
    const int32_t* cu_prefix_host, void* attn_out, const void* logits_steps, int vocab,
    const float* temperature_host, float budget, float stop_entropy, uint64_t seed,
    uint32_t step0, int32_t* canvas, int32_t* canvas_history, int32_t* halt_step, int* steps_run,
    void* workspace, size_t workspace_bytes, dd_stream_t stream);

/* dd_denoise_block_adaptive with the loop kept on the device.  The steps
 * are captured once into a CUDA graph: memset nodes that reset the loop
 * state, then one conditional (IF) node per step, run in order.  A small
 * kernel at the end of each step's body reads the halt flags and sets the
 * next step's condition, to 0 once every canvas has halted, so the
 * remaining steps' bodies are skipped on the device.  No step waits for the
 * host.
 *   dd_denoise_block_adaptive_graph_create captures the loop with exactly
 *     these arguments (those of dd_denoise_block_adaptive, without the
 *     stream, with steps_run a DEVICE int32 written by the graph) and
 *     instantiates it.  It validates like dd_denoise_block_adaptive,
 *     launches nothing and stores a handle in *out (NULL on failure).
 *   dd_denoise_block_adaptive_graph_launch replays it on `stream`.  The
 *     results (canvas, canvas_history rows 0 .. steps_run - 1, halt_step,
 *     *steps_run) equal those of the eager call with the same arguments.
 *     dd_launch_count counts every kernel of every step body per replay,
 *     an upper bound, as the bodies skipped on the device are not known to
 *     the host.  Buffers must stay allocated while the handle exists, and
 *     replays that may overlap in time must not share a workspace.
 *   dd_denoise_block_adaptive_graph_destroy frees it (NULL is accepted). */
typedef struct dd_adaptive_graph_st* dd_adaptive_graph;
DD_API dd_status dd_denoise_block_adaptive_graph_create(
    dd_adaptive_graph* out, const dd_attn_desc* desc, int max_steps, const void* q_steps,
    const void* kc_steps, const void* vc_steps, const void* k_prefix, const void* v_prefix,
    const int32_t* cu_prefix, const int32_t* cu_prefix_host, void* attn_out,
    const void* logits_steps, int vocab, const float* temperature_host, float budget,
    float stop_entropy, uint64_t seed, uint32_t step0, int32_t* canvas, int32_t* canvas_history,
    int32_t* halt_step, int32_t* steps_run, void* workspace, size_t workspace_bytes);
DD_API dd_status dd_denoise_block_adaptive_graph_launch(dd_adaptive_graph graph,
                                                        dd_stream_t stream);
DD_API dd_status dd_denoise_block_adaptive_graph_destroy(dd_adaptive_graph graph);

/* Clears a whole workspace: the error word and the sampler's state (async on
 * stream).  Call once before a workspace's first use. */
DD_API dd_status dd_workspace_init(void* workspace, size_t workspace_bytes, dd_stream_t stream);

/* Synchronises `stream`, reads the workspace's latched device error and
 * clears it.  Returns DD_OK, DD_ERR_DEVICE_TIMEOUT or DD_ERR_DEVICE_BOUNDS. */
DD_API dd_status dd_query_device_error(void* workspace, dd_stream_t stream);

/* Static description of a status code. */
DD_API const char* dd_status_string(dd_status status);

/* Detail of the last failure on this host thread ("" if none). */
DD_API const char* dd_last_error(void);

/* Test hook for the device-timeout path (the pages have no counterpart).
 * Every wait of the tensor-core kernels (attention, soft embedding, MLP) on
 * an mbarrier is bounded in time.  With ns != 0, the kernels launched
 * afterwards from this host thread make one extra wait, once their first
 * MMAs are in flight, on an mbarrier that nothing completes, and their
 * pipeline waits are limited to ns nanoseconds: the wait runs out, the call
 * latches DD_ERR_DEVICE_TIMEOUT in its workspace (read it with
 * dd_query_device_error), and every CTA waits (up to 1 s per wait) for its
 * own copies and MMAs in flight, frees its tensor memory and returns.  The
 * outputs of such a call are undefined; clear the workspace
 * (dd_workspace_init) before its next use.  ns = 0 (the default) turns the
 * stall off. */
DD_API void dd_set_test_stall_ns(uint64_t ns);

/* Number of kernels the library launched on this host thread since the last
 * call to dd_reset_launch_count (for launch accounting in benchmarks). */
DD_API uint64_t dd_launch_count(void);
DD_API void dd_reset_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DD_H_ */

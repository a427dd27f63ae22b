/* libgpt2: one GPT-2 training step on one NVIDIA B200 (sm_100a).
 *
 * C ABI: plain pointers and sizes only.  "d_" arguments are device pointers
 * (CUDA global memory on the current device), "h_" arguments host pointers.
 * Every call returns a status code (GPT2_OK = 0 or a negative GPT2_E*) unless
 * documented otherwise; gpt2_last_error() gives a one-line reason.  Calls are
 * asynchronous on the handle's stream unless an h_ output is requested, which
 * synchronises that stream.
 *
 * The method (the pages it is described on):
 *  - "Let's reproduce GPT-2 (124M)", video summary, Key Takeaways: the
 *    architecture bullet (decoder-only, pre-LayerNorm, extra final LayerNorm,
 *    GELU, 12 layers x 768 channels, vocab 50,257, seq 1024), the
 *    hyperparameter bullet (AdamW betas 0.9/0.95, eps 1e-8, clip 1.0, weight
 *    decay 0.1 on 2D tensors, warmup + cosine LR), the accumulation bullet
 *    (loss divided by the number of micro-steps) and the weight tying /
 *    padding bullet (tied wte/lm_head, vocab padded 50257 -> 50304).
 *  - "Let's reproduce GPT-2 (124M)", video page, Chapters: cross entropy
 *    loss; parameter sharing wte and lm_head; model initialization (std 0.02,
 *    residual init); AdamW, gradient clipping; gradient accumulation.
 *  - "From Scratch: Building GPT-2 for Efficient Language Modeling", Key
 *    Features (token + positional embeddings, attention, GELU MLP, residuals)
 *    and Training Setup table.
 *
 * Flat parameter order (also the order of grads, AdamW moments and
 * checkpoints), every Linear weight stored [out, in] row-major:
 *   wte[Vp, C], wpe[block, C];
 *   per layer l: ln1.g[C], ln1.b[C], attn.w[3C, C], attn.b[3C], proj.w[C, C],
 *                proj.b[C], ln2.g[C], ln2.b[C], fc.w[4C, C], fc.b[4C],
 *                mproj.w[C, 4C], mproj.b[C];
 *   lnf.g[C], lnf.b[C].
 */
#ifndef GPT2_B200_H
#define GPT2_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPT2_OK 0
#define GPT2_EINVAL (-1)     /* bad argument: null pointer, size out of range, unsupported shape */
#define GPT2_ECUDA (-2)      /* a CUDA runtime call or kernel launch failed, or a device wait timed out */
#define GPT2_ETOKEN (-3)     /* a token or target id outside [0, padded_vocab) (flagged on the device) */
#define GPT2_ENOMEM (-4)     /* device or host allocation failed */
#define GPT2_ESTATE (-5)     /* call out of order (e.g. backward without a forward with targets) */
#define GPT2_ENONFINITE (-6) /* non-finite gradient norm: the AdamW update was skipped */

#define GPT2_FP32 0 /* fp32 everywhere, CUDA-core (FFMA) matmuls: the parity mode */
#define GPT2_BF16 1 /* bf16 tensor-core matmuls and attention, fp32 master weights,
                       fp32 residual stream, fp32 LayerNorm statistics, LSE and loss */

typedef struct {
  int n_layer;      /* number of blocks L */
  int n_head;       /* attention heads H (head dim C/H; must be 64 in BF16 mode) */
  int n_embd;       /* channels C (multiple of 128, at most 1024) */
  int vocab_size;   /* real vocabulary (targets must lie below it in practice) */
  int padded_vocab; /* rows of wte = logits columns Vp (multiple of 64, at most 65472; 51200 in FP32 mode) */
  int block_size;   /* maximum sequence length (rows of wpe) */
  int max_B;        /* largest micro-batch the activations are sized for */
  int max_T;        /* largest sequence length the activations are sized for (<= block_size) */
  int precision;    /* GPT2_FP32 or GPT2_BF16 */
} gpt2_config;

typedef struct gpt2 gpt2_t; /* opaque; the library owns every device buffer it allocates */

/* Allocate parameters, gradients, AdamW moments and activations on the
 * current device and initialise the weights on the device from `seed`
 * (counter-based normal generator): matrices and embeddings N(0, 0.02), the two
 * residual projections N(0, 0.02/sqrt(2L)), biases 0, LayerNorm gains 1 and
 * shifts 0 ("Let's reproduce GPT-2 (124M)", Chapters: model initialization).
 * Gradients and moments start at zero.  *out receives the handle. */
int gpt2_create(const gpt2_config* cfg, uint64_t seed, gpt2_t** out);
/* Free everything the handle owns (synchronises its stream).  NULL is a no-op. */
void gpt2_destroy(gpt2_t* h);
/* Enqueue all later work on `cuda_stream` (a cudaStream_t; NULL = legacy default stream). */
int gpt2_set_stream(gpt2_t* h, void* cuda_stream);

/* Forward pass on d_tokens[B*T] (int32, row-major [B, T], device memory the
 * caller keeps alive until the stream reaches it).  With d_targets non-NULL,
 * also the mean softmax cross-entropy over all B*T positions and all Vp
 * columns, the per-row argmax, and the state that gpt2_backward needs; with
 * NULL, logits only.  B <= max_B, T <= max_T.  h_loss non-NULL: the loss is
 * copied out (syncs; an out-of-range id then returns GPT2_ETOKEN). */
int gpt2_forward(gpt2_t* h, const int32_t* d_tokens, const int32_t* d_targets, int B, int T, float* h_loss);
/* Backward pass of the last forward-with-targets, scaling the loss by
 * loss_scale (1/accumulation steps): every gradient += d(loss*loss_scale)/dparam
 * ("Let's reproduce GPT-2 (124M)", Key Takeaways: gradient accumulation).
 * The tied wte gradient receives both its lm_head and its embedding terms. */
int gpt2_backward(gpt2_t* h, float loss_scale);
/* Forward with targets and backward in one call, with the softmax gradient
 * written in the same pass over the logits as the loss (the logits buffer is
 * overwritten by its gradient, so gpt2_get_logits is unavailable after it). */
int gpt2_forward_backward(gpt2_t* h, const int32_t* d_tokens, const int32_t* d_targets, int B, int T,
                          float loss_scale, float* h_loss);
/* Set every gradient to zero. */
int gpt2_zero_grad(gpt2_t* h);
/* CUDA-graph replay of gpt2_forward_backward / gpt2_train_step micro-steps
 * (default: enabled).  The kernel sequence of a (B, T, loss_scale)
 * combination is captured the second time it is used and replayed afterwards,
 * on a private stream ordered after the handle's stream; results are identical
 * to eager launches.  Never used while timing is enabled. */
int gpt2_set_graphs(gpt2_t* h, int enable);
/* Global-norm clip then AdamW ("Let's reproduce GPT-2 (124M)", Key Takeaways:
 * optimization hyperparameters): n = ||g||_2 over all parameters (tied wte
 * once), s = min(1, clip/(n + 1e-6)), g' = s*g; step t += 1;
 * p *= 1 - lr*wd on 2D tensors (wte, wpe, Linear weights) only;
 * m = b1 m + (1-b1) g'; v = b2 v + (1-b2) g'^2;
 * p -= lr * (m/(1-b1^t)) / (sqrt(v/(1-b2^t)) + eps).
 * A non-finite n leaves parameters, moments and t unchanged; it is reported
 * as GPT2_ENONFINITE by this call when h_grad_norm is non-NULL (syncs) and
 * otherwise by the next call that syncs.  h_grad_norm receives n. */
int gpt2_adamw_step(gpt2_t* h, float lr, float wd, float b1, float b2, float eps, float clip, float* h_grad_norm);
/* One whole optimizer step from HOST token buffers: zero_grad, then for each
 * of n_micro micro-steps copy h_tokens/h_targets[k*B*T .. (k+1)*B*T) to the
 * device and run forward+backward with loss_scale 1/n_micro, then
 * gpt2_adamw_step.  h_loss receives the mean micro-step loss and h_grad_norm
 * the pre-clip norm (both may be NULL; either one syncs). */
int gpt2_train_step(gpt2_t* h, const int32_t* h_tokens, const int32_t* h_targets, int n_micro, int B, int T,
                    float lr, float wd, float b1, float b2, float eps, float clip, float* h_loss,
                    float* h_grad_norm);
/* Learning rate at step `it`: linear warmup max_lr*(it+1)/warmup for it <
 * warmup, min_lr after max_steps, cosine from max_lr to min_lr in between
 * ("Let's reproduce GPT-2 (124M)", Chapters: learning rate scheduler; "From
 * Scratch: Building GPT-2", Training Setup: 715 warmup steps, 19073 iterations). */
double gpt2_lr_at(int it, double max_lr, double min_lr, int warmup, int max_steps);

/* ---- generation (forward only, KV cache; bf16 mode) ----
 * "Let's reproduce GPT-2 (124M)", Chapters: sampling init, prefix tokens;
 * sampling loop.  The model continues B prefixes of equal length one token
 * at a time.  The cache holds every layer's keys and values for up to
 * block_size positions of max_B sequences (allocated by the first prefill:
 * n_layer * max_B * block_size * 2 * n_embd bf16).
 * Next-token rule: top-k sampling from softmax(logits / temperature) over the
 * top_k largest logits of the real vocabulary [0, vocab_size) (ties at the
 * k-th place to the lower id); top_k = 1 or temperature = 0 is the greedy
 * argmax.  The uniform draw of sequence b for the token at position p is the
 * top 53 bits of splitmix64(seed * 2^32 + p * 2^16 + b), where splitmix64 is
 * the generator of Steele, Lea and Flood (OOPSLA 2014), so every draw is
 * reproducible.  1 <= top_k <= 64; GPT2_EINVAL otherwise or in FP32 mode.
 * d_next: device int32 [B] that receives the next token of every sequence. */
/* Run the forward on d_tokens [B, T0] (T0 <= max_T), fill the cache with
 * positions 0..T0-1 and sample the token at position T0 from the last
 * position's logits.  Replaces whatever the cache held. */
int gpt2_prefill(gpt2_t* h, const int32_t* d_tokens, int B, int T0, float temperature, int top_k, uint64_t seed,
                 int32_t* d_next);
/* One step: d_tokens [B] are the tokens at position pos, which must equal the
 * number of positions the cache holds (T0 after the prefill, +1 per step) and
 * be below block_size; B must be the prefill's.  Appends their keys and values
 * to the cache and samples the token at position pos + 1. */
int gpt2_decode_step(gpt2_t* h, const int32_t* d_tokens, int B, int pos, float temperature, int top_k,
                     uint64_t seed, int32_t* d_next);
/* [B, Vp] logits (as fp32) from which the last prefill or decode step drew. */
int gpt2_get_decode_logits(gpt2_t* h, float* h_dst);

/* ---- accessors (parity checks, checkpoint / resume); all synchronise ---- */
int64_t gpt2_num_params(const gpt2_t* h);
int gpt2_get_params(gpt2_t* h, float* h_dst);       /* fp32 master weights, flat order */
int gpt2_set_params(gpt2_t* h, const float* h_src); /* also refreshes the bf16 copy */
int gpt2_get_grads(gpt2_t* h, float* h_dst);
int gpt2_get_adam_state(gpt2_t* h, float* h_m, float* h_v, int64_t* h_step); /* any may be NULL */
int gpt2_set_adam_state(gpt2_t* h, const float* h_m, const float* h_v, int64_t step);
int gpt2_get_logits(gpt2_t* h, float* h_dst);  /* [B, T, Vp] of the last forward, as fp32 */
int gpt2_get_argmax(gpt2_t* h, int32_t* h_dst); /* [B, T], lowest index among maxima */
int gpt2_get_losses(gpt2_t* h, float* h_dst);   /* [B, T] per-position losses of the last forward */
int gpt2_last_loss(gpt2_t* h, float* h_loss);   /* mean loss of the last forward with targets */
/* Sorted (token << 16 | position) keys of the last backward's embedding
 * scatter-add ([B*T] uint32, BF16 and FP32 modes). */
int gpt2_get_embed_keys(gpt2_t* h, uint32_t* h_dst);
/* Number of kernels this handle has launched since creation. */
int64_t gpt2_kernel_launches(const gpt2_t* h);
/* Guard bytes (no counterpart in the paper: a check of this library's own
 * kernels).  Every device buffer the handle allocates is rounded up to 256
 * bytes and followed by 256 guard bytes of 0xA5.  Waits for the handle's
 * work, then *n_bad = the number of guard bytes that no longer hold 0xA5
 * (0 unless some kernel wrote past the end of a buffer). */
int gpt2_check_guards(gpt2_t* h, int64_t* n_bad);
/* Test hook for the check above: overwrites one byte of the guard of the
 * index-th allocation (in allocation order).  GPT2_EINVAL for an index out of
 * range. */
int gpt2_debug_overwrite_guard(gpt2_t* h, int index);

/* ---- measurement support ----
 * With timing enabled, every operation this handle enqueues is bracketed by a
 * pair of CUDA events on the handle's stream and its device time is
 * accumulated per kernel class, together with the operation's algorithmic
 * work: FLOPs (2*M*N*K for a matrix product, 4*B*H*d*(causal score count) for
 * attention forward, twice that for its backward) and the bytes an ideal
 * kernel must move through HBM.  Classes (array index):
 *   0 matmul (tcgen05 GEMM and its split-K reduction)  1 attention forward
 *   2 attention backward  3 LayerNorm forward  4 LayerNorm backward (+ bias sums)
 *   5 cross-entropy  6 gradient norm + AdamW  7 embedding  8 other (colsum, loss mean) */
#define GPT2_NUM_KCLASSES 9
int gpt2_set_timing(gpt2_t* h, int enable);
/* Synchronise, then fill h_ms / h_ops / h_flops / h_bytes (arrays of
 * GPT2_NUM_KCLASSES; any may be NULL) with the totals since the last call, and
 * reset them.  h_ops counts timed operations (one or two kernels each). */
int gpt2_get_timing(gpt2_t* h, double* h_ms, int64_t* h_ops, double* h_flops, double* h_bytes);
/* One-line description of the last failure on this handle (never NULL). */
const char* gpt2_last_error(const gpt2_t* h);

/* ---- standalone operators (device pointers, caller-owned memory) ---- */

/* Causal multi-head attention forward, bf16, head dim 64, softmax scale
 * 1/sqrt(64) ("Let's reproduce GPT-2 (124M)", Key Takeaways: architecture and
 * flash attention bullets).  d_qkv: [B, T, 3C] bf16 with q, k, v the column
 * blocks [0,C), [C,2C), [2C,3C) and head h in columns h*64..h*64+63 of each
 * (C = 64*H).  d_out: [B, T, C] bf16.  d_lse: [B, H, T] fp32 natural-log
 * softmax denominators.  Returns GPT2_EINVAL for non-positive sizes or
 * pointers not 16-byte aligned, and when B*H exceeds 65535 (one grid row
 * per (batch, head)). */
int gpt2_attention_forward(const void* d_qkv, void* d_out, float* d_lse, int B, int T, int H, void* cuda_stream);
/* Backward of gpt2_attention_forward: d_dqkv [B, T, 3C] bf16 receives dq, dk,
 * dv in the same column layout.  d_work: caller-provided fp32 scratch of at
 * least gpt2_attention_workspace_floats(B, T, H) elements, 16-byte aligned:
 * lse*log2(e) and D = rowsum(dO * O) for every query, in whole blocks of 128
 * queries (2*B*H*ceil(T/128)*128 floats), then the bf16 dS = P * (dP - D)
 * tiles of 128 x 128 for every (batch, head, query block, key block at or
 * below it) (B*H*n*(n+1)/2 tiles, n = ceil(T/128), 32 KB each).  dS is formed
 * once per score by the dK/dV kernel and read back for dQ.  Deterministic:
 * the same inputs give the same bits. */
int gpt2_attention_backward(const void* d_qkv, const void* d_out, const void* d_dout, const float* d_lse,
                            void* d_dqkv, float* d_work, int B, int T, int H, void* cuda_stream);
int64_t gpt2_attention_workspace_floats(int B, int T, int H);

/* bf16 tensor-core matrix product D[M,N] = sum_k A[m,k] B[n,k] (fp32
 * accumulate) with a fused epilogue, the contraction every Linear layer of the
 * model reduces to.  a_mn = 0: A stored [M][lda] (k contiguous), 1: [K][lda]
 * (m contiguous); b_mn likewise for B ([N][ldb] or [K][ldb]).  epi:
 *   0 out bf16 = D (+bias)          1 out fp32 = D (+bias)
 *   2 out fp32 = resid + D (+bias)  3 out bf16 = u = D + bias, out2 bf16 = gelu_tanh(u)
 *   4 out bf16 = D * gelu_tanh'(aux bf16)
 *   5 out fp32 += D (split over K into d_work when d_work is non-NULL and large enough)
 * out, resid, aux are [M][ldc].  lda, ldb, ldc multiples of 8; A, B, out
 * 16-byte aligned.  bias: fp32 [N] or NULL.  GPT2_EINVAL otherwise. */
int gpt2_matmul_bf16(const void* d_A, int64_t lda, int a_mn, const void* d_B, int64_t ldb, int b_mn, int M, int N,
                     int K, int epi, const float* d_bias, const float* d_resid, void* d_out, void* d_out2,
                     const void* d_aux, int64_t ldc, float* d_work, size_t work_bytes, void* cuda_stream);
/* Bytes of d_work with which an epi = 5 call of this shape splits over K. */
size_t gpt2_matmul_workspace_bytes(int M, int N, int K);

/* ---- device-side errors of the standalone operators ----
 * The kernels never trap.  A pipeline wait that gives up (a producer or
 * consumer that did not arrive within the wait limit) records an error code
 * in a per-device error word and the kernel returns early, leaving its outputs
 * incomplete.  The model handle's syncing calls read that word themselves; the
 * standalone operators above (and gpt2_attention_backward_noalloc below) are
 * asynchronous and do not, so callers check it here:
 * gpt2_check_device_error synchronises cuda_stream (NULL = legacy default
 * stream), then reads and clears the error word of the current device.
 * Returns GPT2_OK when no kernel recorded an error since the last check, and
 * GPT2_ECUDA when one did (or the synchronisation failed).  The word is shared
 * by every caller on the device: check before trusting a standalone result. */
int gpt2_check_device_error(void* cuda_stream);
/* Testing support: the time after which a device-side pipeline wait gives up,
 * in nanoseconds (0 restores the default of 2 s), on the current device.  The
 * waits with which a kernel drains its own in-flight copies and MMAs before
 * returning keep a fixed 2 s limit, so a shortened limit makes kernels give up
 * early and return cleanly; it never leaves work in flight. */
int gpt2_set_wait_limit_ns(uint64_t limit_ns);

/* ---- attention backward without any allocation ----
 * (No counterpart in the paper: this is a calling convenience of this library.)
 * The same computation as gpt2_attention_backward, for callers that cannot
 * call cudaMalloc and have no spare device buffer to hand over as d_work: for
 * example a host framework that plans every byte of device memory ahead of
 * time and forbids allocations outside its planner, or a process that runs
 * with the device memory already fully reserved.  Its scratch (two fp32 per
 * (batch, head, position) row, rows padded to whole blocks of 128 positions)
 * lives in a fixed array inside the library of 2 * GPT2_ATTN_NOALLOC_MAX_ROWS
 * floats (4 MiB); every GPU that loads the library holds that array until the
 * process exits.  Having no room for the dS tiles, it forms dQ from scores
 * recomputed in a dQ kernel of its own instead of reading dS back; that kernel
 * does the same arithmetic on every score in the same order.
 *  - B*H*ceil(T/128)*128 must be at most GPT2_ATTN_NOALLOC_MAX_ROWS and B*H at
 *    most 65535, else GPT2_EINVAL and nothing is enqueued.  Other arguments as
 *    for gpt2_attention_backward, whose results it reproduces bit for bit.
 *  - Like the other standalone operators it is asynchronous: a kernel that
 *    gave up on a wait is reported by gpt2_check_device_error (above), not by
 *    this call's return value.
 *  - The first call on each device looks up the array's device address on
 *    that device (with it current); make that first call before any stream
 *    capture.  No call allocates device or host memory.
 *  - All calls share the one array and it keeps the last call's contents; the
 *    kernels overwrite every scratch element they read, so nothing needs to be
 *    cleared.  Calls that overlap on the GPU (different streams, or different
 *    host threads on one device) race on the array: serialise them. */
#define GPT2_ATTN_NOALLOC_MAX_ROWS (1 << 19)
int gpt2_attention_backward_noalloc(const void* d_qkv, const void* d_out, const void* d_dout, const float* d_lse,
                                    void* d_dqkv, int B, int T, int H, void* cuda_stream);

#ifdef __cplusplus
}
#endif
#endif /* GPT2_B200_H */

/*
 * nc.h -- C ABI of the B200 (sm_100a) nanochat base-pretraining step.
 *
 * The step is the one the dev.to guide "Como treinar seu proprio ChatGPT
 * por 50 dolares" describes for scripts.base_train: forward and backward
 * of the depth-parametrised GPT of its section "1. Modelo GPT
 * (nanochat/gpt.py)" under next-token cross-entropy, then the Muon update
 * of the 2-D block matrices of its section "2. Otimizador Muon
 * (nanochat/optim.py)".  --depth selects every shape (section "Filosofia:
 * Um Unico Seletor Para Controlar Tudo"): d = 64*depth, head_dim 128
 * (one head of width d when d < 128), MLP width 4d; the BPE vocabulary
 * has 32768 entries (table "O Que o nanochat Abrange").
 *
 * Conventions shared by every entry point:
 *   - Every call returns nc_status; nothing throws or aborts across the ABI.
 *     On failure nc_last_error() returns a thread-local message.
 *   - Work is enqueued on the handle's CUDA stream (nc_set_stream; default:
 *     the legacy default stream).  Calls return before the GPU finishes
 *     unless stated otherwise.
 *   - Objects (nc_params, nc_grads) are owned by the library and released
 *     with the matching *_free.  Pointers passed in are borrowed.
 *   - "host or device" pointer arguments are classified with
 *     cudaPointerGetAttributes; host memory is copied in or out on the
 *     handle's stream.
 *   - Bounded device waits: a kernel that waits too long on an mbarrier
 *     records NC_ERR_TIMEOUT in a device status word instead of hanging;
 *     the next synchronising call returns it and the handle is poisoned.
 *   - Matrices are row-major [out, in] (y = x W^T).  bf16 is IEEE bfloat16
 *     with round-to-nearest-even; accumulation is fp32.
 */
#ifndef NC_H
#define NC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NC_OK = 0,
  NC_ERR_INVALID_ARG = 1, /* bad size, null pointer, unsupported shape      */
  NC_ERR_OOM = 2,         /* device allocation failed                       */
  NC_ERR_CUDA = 3,        /* a CUDA runtime call failed                     */
  NC_ERR_TOKEN_RANGE = 4, /* a token or target id outside [0, vocab)        */
  NC_ERR_TIMEOUT = 5,     /* a bounded device wait expired; handle poisoned */
  NC_ERR_UNSUPPORTED = 6  /* valid request this library does not implement  */
} nc_status;

typedef enum { NC_F32 = 0, NC_BF16 = 1, NC_I32 = 2 } nc_dtype;

typedef struct nc_params nc_params;
typedef struct nc_grads nc_grads;

/* One parameter or gradient tensor.  data: device pointer of the fp32
 * storage (parameters: the fp32 master; gradients: the fp32 gradient).
 * data_bf16: device pointer of the bf16 working copy the kernels read
 * (NULL for the embedding, which is gathered from the fp32 master). */
typedef struct {
  char name[32];
  int ndim;
  int64_t shape[2];
  nc_dtype dtype;
  void* data;
  void* data_bf16;
} nc_tensor_desc;

/* ------------------------------------------------------------------ model */

/* Flags of nc_gpt_init_ex. */
#define NC_INIT_SPEC 0        /* out-projections (wo, wdown) and lm_head zero */
#define NC_INIT_ALL_RANDOM 1  /* every tensor random; lm_head std 1/sqrt(d)   */

/* Create a model of the given depth on the current CUDA device and draw its
 * weights from seed: N(0, 1/fan_in) for every matrix (std 1 for the
 * embedding), out-projections and lm_head zero (guide, section "1. Modelo
 * GPT"; the zero out-projections as the workload fixes them).  Normals come
 * from a counter-based SplitMix64 stream and Box-Muller: element i of
 * tensor t uses splitmix64(key_t + 2i) and splitmix64(key_t + 2i + 1),
 * key_t = splitmix64(seed ^ splitmix64(t + 1)).
 * depth: an even number in [2, 32] (head_dim 128, at most 16 heads; depth 1,
 * whose single head is 64 wide, returns NC_ERR_UNSUPPORTED);
 * vocab: [8, 32768], multiple of 8.
 * Parameters, Muon momentum (zero) and bf16 copies are allocated here;
 * activations are allocated by the first nc_gpt_fwd_bwd of a given B*T.
 * Synchronises the device before returning.
 * Errors: NC_ERR_INVALID_ARG (depth/vocab), NC_ERR_OOM, NC_ERR_CUDA. */
nc_status nc_gpt_init(int depth, int vocab, uint64_t seed, nc_params** out);
nc_status nc_gpt_init_ex(int depth, int vocab, uint64_t seed, int flags, nc_params** out);

/* Model variants of the guide's section "1. Modelo GPT": fewer KV heads
 * ("GQA") and attention windows that alternate short and long context
 * across layers (the "SSSL" pattern, passed to the attention call as its
 * window_size).
 *   n_kv_head: 0 = one KV head per query head (the default model); else it
 *     must divide n_head = d / 128.  wk and wv then have n_kv_head * 128
 *     rows, and query head h reads KV head h / (n_head / n_kv_head).
 *   window: NULL = full causal attention in every layer; else `depth`
 *     entries (borrowed, read during this call only): layer l lets query t
 *     see keys t - window[l] .. t; a negative entry is full causal.  A
 *     pattern string maps to it as layer l taking the pattern's letter
 *     l % length, 'S' a short window, 'L' full causal.
 * depth, vocab, seed and flags as for nc_gpt_init_ex.  Errors: as
 * nc_gpt_init_ex, and NC_ERR_INVALID_ARG for an n_kv_head that does not
 * divide n_head. */
typedef struct {
  int depth, vocab;
  uint64_t seed;
  int flags;
  int n_kv_head;
  const int32_t* window;
  /* Non-zero: the guide's "--fp8" training (section "1. Modelo GPT"): every
   * GEMM of the block projections (q|k|v, o, up, down; forward, input and
   * weight gradients) runs on E4M3 operands, each operand tensor quantised
   * whole with its own dynamic scale (nc_op_fp8_quantize; wq|wk|wv as one
   * tensor, weights from their fp32 masters), the products dequantised in
   * the GEMM epilogue; lm_head, attention and the norms stay as they are.
   * Needs d >= 256 (NC_ERR_UNSUPPORTED) and B*T > 128, a multiple of 16
   * (NC_ERR_INVALID_ARG from the step). */
  int fp8;
  /* The untied lm_head (guide, section "1. Modelo GPT") and the softmax
   * cross-entropy in chunks of this many tokens: each chunk's logits are
   * computed, turned into their loss rows and, in place, their gradient,
   * and consumed by the lm_head weight and input gradients before the next
   * chunk, so only chunk x vocab bf16 logits are held.  0: 32768 tokens (a
   * 2 GB logits buffer at vocab 32768; at depth 20, B = 32, T = 2048 it ran
   * about 1 ms faster per step than one 65536-token chunk).  Results do not
   * depend on it beyond fp32 summation order in the lm_head weight
   * gradient. */
  int lm_chunk_tokens;
} nc_model_config;
nc_status nc_gpt_init_config(const nc_model_config* cfg, nc_params** out);
void nc_params_free(nc_params* p);

/* Stream all later work of this handle is enqueued on (a cudaStream_t). */
nc_status nc_set_stream(nc_params* p, void* cuda_stream);

/* Number of parameter tensors (6*depth + 2) and their descriptors, in the
 * order: wte [V,d]; per layer wq, wk, wv, wo [d,d], wup [4d,d],
 * wdown [d,4d]; lm_head [V,d].  wq, wk, wv of a layer are adjacent in
 * memory (one [3d, d] matrix).  With n_kv_head set (nc_gpt_init_config),
 * wk and wv are [128 n_kv_head, d] and the three form one
 * [d + 256 n_kv_head, d] matrix. */
int nc_num_tensors(const nc_params* p);
nc_status nc_tensor_info(const nc_params* p, int idx, nc_tensor_desc* out);

/* Re-derive every bf16 working copy from the fp32 masters (call after
 * writing masters through nc_tensor_info pointers). */
nc_status nc_params_sync(nc_params* p);

/* Copy the fp32 master of parameter idx in from `src` or out to `dst`
 * (host or device pointer, shape[0]*shape[1] floats); writing also
 * refreshes that tensor's bf16 copy.  Both synchronise the stream.
 * Errors: NC_ERR_INVALID_ARG (index, null), NC_ERR_CUDA. */
nc_status nc_tensor_write(nc_params* p, int idx, const float* src);
nc_status nc_tensor_read(const nc_params* p, int idx, float* dst);

/* Muon momentum buffer of block matrix idx (1 <= idx <= 6*depth), fp32,
 * copied out to `dst` (host or device).  Synchronises. */
nc_status nc_momentum_read(const nc_params* p, int idx, float* dst);

/* Gradient buffers (fp32, one per parameter tensor, same order). */
nc_status nc_grads_create(const nc_params* p, nc_grads** out);
void nc_grads_free(nc_grads* g);
nc_status nc_grad_info(const nc_grads* g, int idx, nc_tensor_desc* out);
/* Copy gradient idx out to `dst` / in from `src` (host or device, fp32).
 * Writing lets a caller run nc_muon_step on gradients it computed itself.
 * Both synchronise. */
nc_status nc_grad_read(const nc_grads* g, int idx, float* dst);
nc_status nc_grad_write(nc_grads* g, int idx, const float* src);

/* Forward + backward of the whole model on one batch.
 * tokens, targets: [B, T] int32 row-major, host or device; ids in
 * [0, vocab).  loss_host: host float, receives the mean next-token
 * cross-entropy (natural log) over all B*T positions; this call
 * synchronises the stream to deliver it.  Every gradient in g is
 * OVERWRITTEN (not accumulated).  T must be >= 1 and B*T <= 2^24;
 * activations for B*T tokens are (re)allocated on first use.
 * Errors: NC_ERR_INVALID_ARG, NC_ERR_TOKEN_RANGE (ids are clamped for the
 * reads, so nothing is read out of bounds), NC_ERR_OOM, NC_ERR_TIMEOUT,
 * NC_ERR_CUDA. */
nc_status nc_gpt_fwd_bwd(nc_params* p, const int32_t* tokens, const int32_t* targets, int B,
                         int T, float* loss_host, nc_grads* g);

/* Same, without the synchronisation: the loss is written to loss_dev
 * (device float) and errors found on the device surface at the next
 * synchronising call (nc_sync). */
nc_status nc_gpt_fwd_bwd_async(nc_params* p, const int32_t* tokens, const int32_t* targets, int B,
                               int T, float* loss_dev, nc_grads* g);

/* Muon step on the 6*depth block matrices (guide, section "2. Otimizador
 * Muon"): M <- momentum*M + G; X = M / (||M||_F + 1e-7), transposed to
 * rows <= cols; five Newton-Schulz steps A = X X^T, B = b A + c A A,
 * X = a X + B X with (a, b, c) = (3.4445, -4.7750, 2.0315) in bf16 with
 * fp32 accumulation; W <- W - lr * X (transposed back).  The embedding and
 * lm_head are not touched (the guide gives them to AdamW).  Asynchronous. */
nc_status nc_muon_step(nc_params* p, const nc_grads* g, float lr, float momentum);

/* The step as one CUDA graph.  nc_step_capture records, without running
 * it, one nc_gpt_fwd_bwd_async(p, tokens, targets, B, T, loss_dev, g)
 * followed by nc_muon_step(p, g, lr, momentum) on the handle's stream into
 * a graph the handle owns (replacing an earlier one); nc_step_replay
 * launches that graph on the handle's stream.  A replay reads the token and
 * target buffers given at capture (refill them in place between replays),
 * writes the loss to loss_dev and updates the weights, exactly like the two
 * calls it recorded.  tokens, targets, loss_dev: device memory that must
 * outlive the graph; the handle needs a non-default stream (nc_set_stream).
 * Activations for B*T tokens are allocated before the capture; a later call
 * that reallocates them (another B*T) or the RoPE table (a longer T), or
 * freeing g, releases the graph.  Profiling is paused during the capture;
 * replays add the graph's kernel count to nc_launch_count.
 * Errors: NC_ERR_INVALID_ARG (host pointers, default stream, no captured
 * step), NC_ERR_TIMEOUT (poisoned handle), NC_ERR_OOM, NC_ERR_CUDA. */
nc_status nc_step_capture(nc_params* p, const int32_t* tokens, const int32_t* targets, int B, int T,
                          float* loss_dev, nc_grads* g, float lr, float momentum);
nc_status nc_step_replay(nc_params* p);

/* AdamW step on the embedding (wte, lr_embed) and lm_head (lr_head) from
 * their gradients in g (guide, section "2. Otimizador Muon": embeddings and
 * lm_head take AdamW; the pages give no hyperparameters, so all are
 * arguments).  With t the number of calls on this handle so far (1 for the
 * first), per element:
 *   m <- beta1 m + (1 - beta1) g;   v <- beta2 v + (1 - beta2) g^2
 *   W <- W - lr ((m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)
 *                + weight_decay W)        (decoupled decay, W before the step)
 * in fp32; lm_head's bf16 working copy is refreshed.  The moments (fp32,
 * 4 * vocab * d floats) are allocated and zeroed by the first call; the
 * block matrices are not touched (nc_muon_step).  Asynchronous.
 * Errors: NC_ERR_INVALID_ARG (null, gradients of another handle,
 * lr / eps / weight_decay < 0, betas outside [0, 1)), NC_ERR_TIMEOUT
 * (poisoned handle), NC_ERR_CUDA. */
nc_status nc_adamw_step(nc_params* p, const nc_grads* g, float lr_embed, float lr_head, float beta1,
                        float beta2, float eps, float weight_decay);

/* Wait for the handle's stream; returns the first device-side error. */
nc_status nc_sync(nc_params* p);

/* Testing hook: device address of the handle's status word (one int, 0 =
 * no error; 1 = an expired bounded wait, 2 = a token id out of range), so a
 * test can plant a device-side error code and check how the host reports
 * it without making any kernel fail.  NULL for a null handle. */
int* nc_debug_status_word(nc_params* p);

/* ------------------------------------------------------------------ ops
 * Single kernels of the step, for kernel-level checks and the
 * Newton-Schulz sweep.  All pointers are device pointers; all calls are
 * asynchronous on `stream` (a cudaStream_t, NULL = legacy default).
 * Argument errors return at once, before anything is launched.  Errors a
 * kernel finds on the device (a bounded wait that expired, which leaves the
 * outputs incomplete; a token id out of range) are recorded in one op
 * status word per device, shared by every nc_op_* call on that device from
 * any stream or thread, and returned by the next nc_op_sync. */

/* Wait for `stream`, then return and clear the device's op status word:
 * NC_OK, NC_ERR_TIMEOUT (an op's bounded wait expired; its outputs are
 * incomplete) or NC_ERR_TOKEN_RANGE.  NC_ERR_CUDA if the wait itself fails. */
nc_status nc_op_sync(void* stream);

/* Testing hook: device address of the current device's op status word (one
 * int, 0 = no error, 1 = an expired wait, 2 = a token id out of range), so a
 * test can plant a code and check how nc_op_sync reports it.  NULL if the
 * address cannot be looked up. */
int* nc_debug_op_status_word(void);

/* Embedding gather, the first step of the forward (guide, section "1. Modelo
 * GPT": token embedding, untied from lm_head): x[i, :] = E[tokens[i], :]
 * for i < n, copied bit for bit (fp32 rows of d floats; E [vocab, d] and x
 * [n, d] dense, 16-byte aligned, d a multiple of 4).  An id outside
 * [0, vocab) is clamped to the nearest valid row for the read (row 0 below,
 * row vocab - 1 above) and recorded as NC_ERR_TOKEN_RANGE for nc_op_sync. */
nc_status nc_op_embed_gather(const int32_t* tokens, int64_t n, const float* E, int vocab, int d,
                             float* x, void* stream);

/* The exponential that the attention backward evaluates on the FMA pipe for
 * one pair of recomputed probabilities in four (the rest, and the forward,
 * use the exponential unit):
 * y[i] ~ 2^x[i] from range reduction x = n + f (n = rint(x)) and a degree-3
 * minimax polynomial for 2^f on [-1/2, 1/2], relative error at most 7.5e-5,
 * for x in [-125, 126); below -125 it returns about 2^-125 (the softmax
 * zeroes masked scores itself).  The softmax is exp(s - max) of the guide's
 * causal attention (section "1. Modelo GPT"); this entry runs the same
 * device function over fp32 device arrays x, y of n elements so that its
 * error can be measured.  NC_ERR_INVALID_ARG for n < 0 or null arrays. */
nc_status nc_op_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/* E4M3 quantisation of one GEMM operand (the guide's "--fp8" training,
 * section "1. Modelo GPT", with one dynamic scale per tensor): for x, a
 * rows x cols matrix of bf16 (x_bf16 != 0) or fp32, row stride ldx,
 *   s = 448 / max |x|  (fp32; 1 when x is all zero; NaN elements skipped),
 *   q[r*ldq + c] = E4M3(x[r, c] * s), or q[c*ldq + r] when transpose != 0,
 * E4M3 the OCP 8-bit format (bias 7, largest 448, subnormals down to 2^-9)
 * rounded to nearest even and saturated to +-448.  s goes to *scale (device
 * float), for nc_gemm_desc.ab_scale.  cols and ldx multiples of 8, rows too
 * when transposing, ldq a multiple of 16 and at least the output row
 * length; x and q 16-byte aligned; scratch is one device word the call
 * overwrites.  NC_ERR_INVALID_ARG otherwise. */
nc_status nc_op_fp8_quantize(const void* x, int x_bf16, int64_t rows, int cols, int64_t ldx, int transpose,
                             void* q, int64_t ldq, float* scale, void* scratch, void* stream);

/* The same quantisation of a bf16 matrix into both layouts in one pass:
 * q[r*cols + c] and qT[c*rows + r] (either may be NULL), the form the fp8
 * model uses for an operand that feeds a GEMM and, transposed, a weight
 * gradient.  rows, cols and ldx multiples of 8; pointers 16-byte aligned. */
nc_status nc_op_fp8_quantize2(const void* x_bf16, int64_t rows, int cols, int64_t ldx, void* q, void* qT,
                              float* scale, void* scratch, void* stream);

/* Epilogues of the GEMM engine. */
typedef enum {
  NC_EPI_STORE_BF16 = 0, /* D(bf16) = alpha*acc                               */
  NC_EPI_STORE_F32 = 1,  /* D(f32)  = alpha*acc                               */
  NC_EPI_RESID_F32 = 2,  /* D(f32)  = aux(f32) + alpha*acc       (residual)   */
  NC_EPI_RELU2 = 3,      /* D(bf16) = max(alpha*acc, 0)^2        (ReLU^2)     */
  NC_EPI_RELU2_BWD = 4,  /* D(bf16) = 2*sqrt(aux(bf16))*alpha*acc (aux = relu(u)^2;
                            sqrt by sqrt.approx, relative error ~2^-23)     */
  NC_EPI_AXPBY_BF16 = 5, /* D(bf16) = alpha*acc + beta*aux(bf16)              */
  NC_EPI_ACC_F32 = 6,    /* D(f32) += alpha*acc                  (atomic)     */
  NC_EPI_ROPE_QKNORM = 7 /* fused q|k|v projection: columns [0, H*128) are H q
                            heads and [H*128, (H+Hkv)*128) Hkv k heads of
                            128, rotated by RoPE at position row % T (pairs
                            i, i + 64) then RMS-normalised per head, rstd
                            written to rstd_q[row * H + h] and
                            rstd_k[row * Hkv + h]; the Hkv v heads after them
                            are stored as is.  D(bf16).  Needs
                            N = (H + 2*Hkv)*128 (Hkv = H when rope_Hkv is 0). */
} nc_epilogue;

/* Batched GEMM on the tcgen05 tensor cores, D[b] = epi(op(A[b]) op(B[b])^T):
 *   acc[m, n] = sum_k A(m, k) * B(n, k)
 * A(m, k) = a_kmajor ? A[m*lda + k] : A[k*lda + m]      (bf16)
 * B(n, k) = b_kmajor ? B[n*ldb + k] : B[k*ldb + n]      (bf16)
 * D[m*ldd + n]; aux[m*ldaux + n]; batch strides in elements.
 * lda, ldb, ldd, ldaux and the batch strides must be multiples of 8
 * elements, A, B 16-byte aligned.  M, N, K >= 1.  split_k >= 1 splits the
 * K loop across CTAs (epilogue must be NC_EPI_ACC_F32 when split_k > 1). */
typedef struct {
  int M, N, K, batch;
  const void* A;
  int64_t lda, stride_a;
  int a_kmajor;
  const void* B;
  int64_t ldb, stride_b;
  int b_kmajor;
  void* D;
  int64_t ldd, stride_d;
  const void* aux;
  int64_t ldaux, stride_aux;
  nc_epilogue epi;
  float alpha, beta;
  int split_k;
  /* NC_EPI_ROPE_QKNORM only: sequence length T, query heads H, cos/sin
   * table (float2 [>= T][64], theta_i(pos) = pos * 10000^(-i/64)) and the
   * two rstd outputs (f32 [M * H] for q, [M * Hkv] for k). */
  int rope_T, rope_H;
  const void* rope_tab;
  float* rstd_q;
  float* rstd_k;
  /* KV heads of the fused projection, 1 <= rope_Hkv <= rope_H; 0 means
   * rope_H (one KV head per query head). */
  int rope_Hkv;
  /* Operand type: 0 bf16; 1 OCP E4M3 (one byte per element, the guide's
   * "--fp8" training, section "1. Modelo GPT", here with one dynamic scale
   * per operand tensor).  E4M3 needs both operands K-major, lda, ldb and
   * the batch strides multiples of 16, alpha = 1, M > 128, N > 128 (it runs
   * on 256-wide column tiles, the last one ragged if need be) and any
   * epilogue but NC_EPI_AXPBY_BF16; the product is multiplied by
   * 1 / (ab_scale[0] * ab_scale[1]), the scales nc_op_fp8_quantize wrote
   * for A and B (two device floats). */
  int ab_type;
  const float* ab_scale;
  /* E4M3 operands, batch 1 and a bf16 epilogue (not the RoPE one) only:
   * when not NULL, max |D| over the bf16 values stored is folded into
   * *amax_out with an integer atomic max on the float's bits (the caller
   * zeroes it first), the amax the output's own fp8 quantisation needs. */
  unsigned* amax_out;
} nc_gemm_desc;
nc_status nc_op_gemm(const nc_gemm_desc* desc, void* stream);

/* Parameter-free RMSNorm: y(bf16) = x(f32) / sqrt(mean(x^2) + 1e-6); rstd(f32). */
nc_status nc_op_rmsnorm(const float* x, int64_t rows, int cols, void* y_bf16, float* rstd,
                        void* stream);

/* Causal attention forward on q, k, v (bf16, [B, T, H, 128] rows of stride
 * ld elements, i.e. slices of the fused [B*T, 3d] qkv activation):
 * o(bf16) [B, T, H, 128] with row stride ldo; lse (f32, natural log)
 * [B, H, T].  Scale 1/sqrt(128). */
nc_status nc_op_attention_fwd(const void* q, const void* k, const void* v, int64_t ld, void* o,
                              int64_t ldo, float* lse, int B, int T, int H, void* stream);

/* Causal attention backward: from dO (bf16, stride ldo) and the forward's
 * O, lse: dq (f32, [B,T,H,128] dense, OVERWRITTEN), dk, dv (bf16, stride
 * ldg).  delta_scratch: f32 [B, H, T] workspace.  Every operand row must be
 * 16-byte aligned (strides multiples of 8 elements) and H <= 16; otherwise
 * NC_ERR_INVALID_ARG / NC_ERR_UNSUPPORTED before anything is launched. */
nc_status nc_op_attention_bwd(const void* q, const void* k, const void* v, int64_t ld,
                              const void* o, const void* dout, int64_t ldo, const float* lse,
                              float* dq, void* dk, void* dv, int64_t ldg, float* delta_scratch,
                              int B, int T, int H, void* stream);

/* Causal attention with grouped KV heads and a left window (guide, section
 * "1. Modelo GPT": "GQA: atencao com menos heads KV" and "atencao de janela:
 * contexto curto/longo alternado (ex: 'SSSL')", passed to flash attention as
 * causal=True with a window_size; the pages give no window length).
 * q, o, dO, dq hold H heads of 128 per row (row strides ldq, ldo; dq dense
 * [B, T, H, 128]); k, v, dk, dv hold Hkv heads (strides ldkv, ldg), H a
 * multiple of Hkv; query head h reads KV head h / (H / Hkv).  Query t sees
 * keys [t - window, t]; window < 0 means every key up to t, and so does
 * any window of T - 1 or more (it runs as unbounded).  With Hkv = H,
 * ldkv = ldq and window < 0 these are nc_op_attention_fwd / _bwd.  Layouts,
 * alignment (16-byte rows) and errors otherwise as those; H <= 16 for the
 * backward. */
nc_status nc_op_attention_fwd_ex(const void* q, int64_t ldq, const void* k, const void* v,
                                 int64_t ldkv, void* o, int64_t ldo, float* lse, int B, int T, int H,
                                 int Hkv, int window, void* stream);
nc_status nc_op_attention_bwd_ex(const void* q, int64_t ldq, const void* k, const void* v,
                                 int64_t ldkv, const void* o, const void* dout, int64_t ldo,
                                 const float* lse, float* dq, void* dk, void* dv, int64_t ldg,
                                 float* delta_scratch, int B, int T, int H, int Hkv, int window,
                                 void* stream);

/* Causal attention backward like nc_op_attention_bwd, for callers that
 * cannot allocate device memory (no cudaMalloc / cudaFree of their own, no
 * workspace they can lend): a caller running while another component owns
 * the whole device-memory budget, a path that must not risk the implicit
 * device synchronisation cudaMalloc and cudaFree can cause, or a caller with
 * nowhere to keep a workspace between calls.  The guide has no counterpart:
 * this is a property of the library, not of the method.
 * The D = rowsum(dO * O) scratch lives in a fixed 4 MiB array inside the
 * library's device image (held on every device that loads the library until
 * the process exits), so B * H * T must not exceed 1048576; larger sizes
 * return NC_ERR_INVALID_ARG before anything is launched.  Nothing is
 * allocated: no cudaMalloc, cudaFree or allocating library routine.
 * The first call on each device looks up the array's device address (with
 * that device current) and should come before any stream capture.  The
 * address is kept for the life of the process, so it stays valid only while
 * that device's primary context does: calls after a cudaDeviceReset are not
 * supported.
 * Every call shares the array and it keeps the last call's contents (each
 * call rewrites the entries it uses before reading them); calls that overlap
 * on the GPU (different streams, or graphs running concurrently) race on it.
 * Inputs, outputs and errors otherwise as nc_op_attention_bwd. */
nc_status nc_op_attention_bwd_noalloc(const void* q, const void* k, const void* v, int64_t ld,
                                      const void* o, const void* dout, int64_t ldo,
                                      const float* lse, float* dq, void* dk, void* dv,
                                      int64_t ldg, int B, int T, int H, void* stream);

/* Newton-Schulz orthogonalisation of `count` matrices [rows, cols] (bf16
 * in and out, dense, batch stride rows*cols): Frobenius normalisation
 * (eps 1e-7) then `steps` quintic steps with the coefficients above, on the
 * wide orientation (a tall stack is transposed in and out).  scratch:
 * device workspace of nc_newton_schulz_scratch_bytes() bytes. */
size_t nc_newton_schulz_scratch_bytes(int count, int rows, int cols);
nc_status nc_op_newton_schulz(const void* x_bf16, void* out_bf16, int count, int rows, int cols,
                              int steps, void* scratch, void* stream);

/* ------------------------------------------------------------------ profiling
 * Per-kernel-class device timing with CUDA events recorded on the launch
 * stream around every launch while enabled. */
typedef struct {
  char name[32];
  int launches;
  double total_ms;
  double flops;  /* algorithmic FLOPs of those launches (tensor kernels) */
  double bytes;  /* algorithmic HBM bytes of those launches (memory kernels) */
} nc_kernel_stat;
nc_status nc_profile_enable(nc_params* p, int on);
/* Collects (synchronising) and resets the statistics; *n = classes written. */
nc_status nc_profile_read(nc_params* p, nc_kernel_stat* out, int max, int* n);

/* Kernels launched by this handle since creation (all classes). */
int64_t nc_launch_count(const nc_params* p);

const char* nc_last_error(void);
const char* nc_status_string(nc_status s);

#ifdef __cplusplus
}
#endif

#endif /* NC_H */

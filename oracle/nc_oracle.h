/*
 * nc_oracle.h -- CPU oracle for the nanochat base-pretraining step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The
 * product path (pretraining_step_b200/) never links, imports or calls it,
 * and shares no code, header, table or constant generator with it.
 *
 * What it computes: a plain, slow, double-precision restatement of
 *   - the pre-norm decoder described in the dev.to guide "Como treinar seu
 *     proprio ChatGPT por 50 dolares", section "1. Modelo GPT
 *     (nanochat/gpt.py)": RoPE, QK normalisation, untied embedding and
 *     lm_head, ReLU^2 MLP, causal softmax attention; with the widths that
 *     --depth selects (section "Filosofia: Um Unico Seletor Para Controlar
 *     Tudo": model_dim = 64*depth, head_dim 128, MLP 4*model_dim,
 *     BPE vocabulary 32768 from the "O Que o nanochat Abrange" table);
 *   - next-token cross-entropy and its gradient by hand-written reverse
 *     mode;
 *   - the Muon step of section "2. Otimizador Muon (nanochat/optim.py)":
 *     momentum, Frobenius normalisation, five quintic Newton-Schulz steps
 *     in the page's form A = X^T X, B = b*A + c*A*A, X = a*X + X*B, with
 *     the constant coefficients (a, b, c) = (3.4445, -4.7750, 2.0315).
 *
 * Readings of points the pages leave open (each is listed with its reason
 * in the design notes of the repository):
 *   RMSNorm eps 1e-6 (also for QK-norm); norms before attention, before
 *   the MLP and before lm_head; RoPE base 10000, half-split pairs (i, i+64),
 *   rotation by +theta; QK-norm after RoPE; heads = d/128 (one head of
 *   width d when d < 128); attention scale 1/sqrt(head_dim); loss = mean
 *   over all B*T positions; heavy-ball momentum M <- mu*M + G; update
 *   W <- W - lr*X with no shape scale and no weight decay.
 *
 * Parameter layout (the interface both sides follow, in this order):
 *   0            wte     [V, d]        token embedding
 *   1 + 6l + 0   wq_l    [d, d]
 *   1 + 6l + 1   wk_l    [d, d]        ([n_kv_head * head_dim, d] in the
 *   1 + 6l + 2   wv_l    [d, d]         grouped-KV variant, the *_ex calls)
 *   1 + 6l + 3   wo_l    [d, d]
 *   1 + 6l + 4   wup_l   [4d, d]
 *   1 + 6l + 5   wdown_l [d, 4d]
 *   6L + 1       lm_head [V, d]
 * Every matrix is row-major [out, in], so y = x * W^T.
 *
 * All functions return 0 on success and a negative value on a bad
 * argument.  No function allocates memory the caller must free.
 */
#ifndef NC_ORACLE_H
#define NC_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Model shape derived from depth (guide, "Filosofia" section).
 * out[0..5] = {d, n_head, head_dim, mlp_dim, n_params_tensors, n_block_matrices}.
 * Returns -1 if depth < 1, vocab < 1 or d is not a multiple of head_dim. */
int oc_dims(int depth, int vocab, int64_t* out);

/* Number of elements of parameter tensor `idx` (layout above), -1 if out of range. */
int64_t oc_param_numel(int depth, int vocab, int idx);

/* Variant with grouped KV heads (guide, section "1. Modelo GPT": "GQA:
 * atencao com menos heads KV").  n_kv_head <= 0 means one KV head per
 * query head (the calls above); otherwise it must divide n_head, and wk,
 * wv have n_kv_head * head_dim rows.  oc_dims_ex also writes
 * out[6] = n_kv_head.  Same return values as above. */
int oc_dims_ex(int depth, int vocab, int n_kv_head, int64_t* out);
int64_t oc_param_numel_ex(int depth, int vocab, int n_kv_head, int idx);

/* SplitMix64 mixing function (Steele, Lea & Flood, OOPSLA 2014), exposed
 * so its published test values can be checked. */
uint64_t oc_splitmix64(uint64_t x);

/* Parameter initialisation from seed, drawing from a counter-based
 * SplitMix64 stream and the Box-Muller transform.  Element i of tensor t
 * takes the two words  splitmix64(key_t + 2i)  and  splitmix64(key_t + 2i + 1)
 * with key_t = splitmix64(seed ^ splitmix64(t + 1)), uniform
 * u = (word >> 11) * 2^-53, and  z = sqrt(-2 ln(1 - u1)) * cos(2 pi u2).
 * Weight = z / sqrt(fan_in) (fan_in = in-features; 1 for wte).
 * spec_zero != 0: wo, wdown and lm_head are zero (the specified init);
 * spec_zero == 0: every tensor is random, lm_head with std 1/sqrt(d).
 * params[i] points to caller-owned float storage of oc_param_numel(i). */
int oc_init_params(int depth, int vocab, uint64_t seed, int spec_zero, float* const* params);
/* Same draw for the grouped-KV layout: tensor t takes the first
 * oc_param_numel_ex(t) numbers of its stream. */
int oc_init_params_ex(int depth, int vocab, int n_kv_head, uint64_t seed, int spec_zero,
                      float* const* params);

/* Parameter-free RMSNorm over rows: y = x / sqrt(mean(x^2) + eps). rstd may be NULL. */
int oc_rmsnorm(const double* x, int64_t rows, int cols, double eps, double* y, double* rstd);

/* Rotary embedding of one head-row of width hd at position pos, in place. */
int oc_rope_row(double* v, int hd, int64_t pos, double base);

/* Causal attention over [B, T, H, hd] tensors (row-major, head-interleaved
 * exactly like the [B*T, d] activations).  o is [B, T, H, hd]; lse [B, H, T]
 * (natural log); probs, if not NULL, is [B, H, T, T] with zeros above the
 * diagonal. */
int oc_attention(const double* q, const double* k, const double* v, int B, int T, int H, int hd,
                 double* o, double* lse, double* probs);

/* Causal attention with grouped KV heads and a left window: query head h
 * reads KV head h / (H / Hkv) (H a multiple of Hkv); query t sees keys
 * j in [t - window, t], every key up to t when window < 0.  q, o:
 * [B, T, H, hd]; k, v: [B, T, Hkv, hd]; lse [B, H, T].  With Hkv = H and
 * window < 0 it is oc_attention. */
int oc_attention_ex(const double* q, const double* k, const double* v, int B, int T, int H, int Hkv,
                    int hd, int window, double* o, double* lse);
/* Its reverse mode: dq [B, T, H, hd], dk, dv [B, T, Hkv, hd], OVERWRITTEN. */
int oc_attention_bwd_ex(const double* q, const double* k, const double* v, const double* lse,
                        const double* dout, int B, int T, int H, int Hkv, int hd, int window,
                        double* dq, double* dk, double* dv);

/* Reverse mode of oc_attention: from dout [B, T, H, hd] and the forward's
 * lse, the gradients dq, dk, dv (same layout), OVERWRITTEN. */
int oc_attention_bwd(const double* q, const double* k, const double* v, const double* lse,
                     const double* dout, int B, int T, int H, int hd, double* dq, double* dk,
                     double* dv);

/* One layer-free piece used by kernel-level checks: y = x * W^T for
 * x [rows, k] and W [n, k]. */
int oc_matmul_nt(const double* x, const double* w, int64_t rows, int64_t n, int64_t k, double* y);

/* Whole-model forward (and backward when grads != NULL).
 * tokens, targets: [B, T] int32 row-major.  params: layout above (float).
 * loss: mean next-token cross-entropy (natural log).
 * grads: same layout, double storage, OVERWRITTEN.
 * logits: optional [B*T, V] output of the final layer.
 * Returns -2 if a token or target is out of [0, V). */
int oc_gpt_fwd_bwd(int depth, int vocab, const float* const* params, const int32_t* tokens,
                   const int32_t* targets, int B, int T, double* loss, double* const* grads,
                   double* logits);

/* Same model with grouped KV heads and a window per layer (guide, section
 * "1. Modelo GPT": fewer KV heads; short and long context alternating
 * across layers, e.g. "SSSL", through the window_size of the attention
 * call).  Layer l attends with oc_attention_ex's window window[l] (negative:
 * full causal); window == NULL is full causal everywhere.  Query head h
 * reads KV head h / (n_head / n_kv_head).  With n_kv_head <= 0 and
 * window == NULL this is oc_gpt_fwd_bwd. */
int oc_gpt_fwd_bwd_ex(int depth, int vocab, int n_kv_head, const int32_t* window,
                      const float* const* params, const int32_t* tokens, const int32_t* targets,
                      int B, int T, double* loss, double* const* grads, double* logits);

/* FP8 ("Treinamento FP8 disponivel via --fp8", guide section "1. Modelo GPT";
 * the pages give no recipe, so this is the reading): the OCP E4M3 format
 * (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
 * largest finite 448, subnormals k * 2^-9).
 * oc_e4m3_round: nearest E4M3 value, ties to the even mantissa, magnitudes
 *   above 448 (infinities too) saturate to 448; NaN stays NaN.
 * Operands are quantised from the values a kernel holds: weights from
 * fp32(t_i), activations and their gradients (bf16 in memory) from
 * bf16(fp32(t_i)) -- the decision taken in the kernel's precision.
 * oc_fp8_scale: per-tensor scale s = 448 / max|v_i| in fp32 arithmetic,
 *   v the source values (act != 0: an activation); 1 if all are zero; -1
 *   on a bad argument.
 * oc_fp8_matmul_nt: y = (Q(x) Q(w)^T) / (s_x s_w) with Q(t)_i =
 *   e4m3(v_i * s_t) (fmt 1) or fp32(t_i) * s_t (fmt 0, scaling alone, no
 *   bf16 step); x [rows, k] an activation, w [n, k] a weight.
 * oc_gpt_fwd_bwd_fp8: oc_gpt_fwd_bwd_ex with every GEMM of the block
 *   projections (forward, input gradient, weight gradient of wq|wk|wv, wo,
 *   wup, wdown) computed that way; the fused q|k|v weight [d + 2 dkv, d]
 *   and its output gradient are one tensor each; attention, the embedding
 *   and lm_head stay exact.  fmt as above. */
double oc_e4m3_round(double x);

/* OpenMP threads of later calls: n > 0 sets them; returns the count in
 * effect (for timing the oracle at one thread and at all cores). */
int oc_threads(int n);
float oc_fp8_scale(const double* x, int64_t n, int act);
int oc_fp8_matmul_nt(const double* x, const double* w, int64_t rows, int64_t n, int64_t k,
                     int fmt, double* y);
int oc_gpt_fwd_bwd_fp8(int depth, int vocab, int n_kv_head, const int32_t* window, int fmt,
                       const float* const* params, const int32_t* tokens, const int32_t* targets,
                       int B, int T, double* loss, double* const* grads, double* logits);

/* Newton-Schulz orthogonalisation of one matrix G [rows, cols]:
 * X = G / (||G||_F + eps_norm), then `steps` iterations of the quintic in
 * the page's right-hand form on the orientation whose Gram X^T X is the
 * smaller one (a wide matrix is transposed first and the result transposed
 * back).  out: [rows, cols]. */
int oc_newton_schulz(const double* G, int rows, int cols, int steps, double a, double b, double c,
                     double eps_norm, double* out);

/* Muon update of one block matrix, in place:
 *   M <- mu*M + G;  O = NS5(M);  W <- W - lr*O.
 * W, M: [rows, cols] double; G: [rows, cols] double. */
int oc_muon_update(double* W, double* M, const double* G, int rows, int cols, double lr, double mu);

/* AdamW step t (t >= 1) on one tensor of n elements, in place (guide,
 * section "2. Otimizador Muon": the embeddings and lm_head take AdamW; the
 * pages give no hyperparameters, so they are arguments).  Decoupled weight
 * decay and bias correction:
 *   m <- b1 m + (1 - b1) g;   v <- b2 v + (1 - b2) g^2
 *   W <- W - lr * ( (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps) + wd * W )
 * where the decay term uses W before this step. */
int oc_adamw_update(double* W, double* m, double* v, const double* g, int64_t n, double lr,
                    double b1, double b2, double eps, double wd, int t);

#ifdef __cplusplus
}
#endif

#endif /* NC_ORACLE_H */

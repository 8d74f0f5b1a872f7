/*
 * gpt.h — C ABI of the B200 GPT pretraining-step library (libgpt.so).
 *
 * One training step of the depth-parameterised GPT decoder described in
 * "¿Cómo Entrenar Tu Propio ChatGPT por $50?" (dev.to): the forward and
 * backward pass of the decoder stack (section "1. Modelo GPT": rotary
 * embeddings, QK normalisation, untied token/output weights, ReLU^2 MLP,
 * causal attention), followed by the optimizer of section "2. Optimizador
 * Muon" (Newton-Schulz "Polar Express" orthogonalised momentum for the 2-D
 * block matrices, AdamW for the embedding and lm_head) with fp32 master
 * weights and bf16 compute (section "3. Gestión de Precisión"; the Portuguese
 * page "Como Treinar Seu Próprio ChatGPT por 50 Dólares?" states the fp32
 * masters explicitly).  Width and heads derive from the depth knob (section
 * "La Filosofía: Un Solo Selector para Controlar Todo"); the vocabulary is
 * 32,768 (section "Lo que nanochat cubre").
 *
 * Conventions for every call:
 *   - Memory is owned by the caller.  The library allocates no device
 *     memory: gpt_workspace_size() reports three byte counts, the caller
 *     allocates them (256-byte aligned device memory) and passes them to
 *     gpt_init().  The context itself is a small host object.
 *   - Calls are asynchronous on the stream given to gpt_init() unless
 *     stated otherwise.  Device-side failures (token ids out of range, an
 *     expired bounded wait) are latched in a device error word and
 *     reported by gpt_check(), which synchronises the stream.
 *   - Status codes: GPT_OK (0) or a negative GPT_E* value; the message of
 *     the last failure on the calling thread is gpt_last_error().  No C++
 *     exception crosses this boundary.
 *   - Matrices are row-major [in, out] (y = x W); the token embedding is
 *     [vocab, d_model].  Tensors exchanged through gpt_get_tensor /
 *     gpt_set_tensor are fp32 device buffers of rows * cols elements.
 */
#ifndef GPT_B200_H
#define GPT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  GPT_OK = 0,
  GPT_EINVAL = -1,    /* bad configuration, pointer, alignment or id */
  GPT_ERANGE = -2,    /* a token or target id outside [0, vocab) reached the device */
  GPT_ETIMEOUT = -3,  /* a bounded device-side wait expired; the step's results are invalid */
  GPT_ECUDA = -4      /* a CUDA runtime call failed */
};

/* Tensor kinds for gpt_get_tensor / gpt_set_tensor. */
enum {
  GPT_KIND_PARAM = 0,  /* fp32 master weight (setting it also refreshes the bf16 copy) */
  GPT_KIND_GRAD = 1,   /* fp32 gradient of the mean loss */
  GPT_KIND_MOM = 2,    /* Muon momentum (block matrices only) */
  GPT_KIND_ADAM_M = 3, /* AdamW first moment (tensors of the AdamW group only) */
  GPT_KIND_ADAM_V = 4, /* AdamW second moment (tensors of the AdamW group only) */
  GPT_KIND_NORMUON_V = 5 /* NorMuon second moment (block matrices only): d
                          * floats, one per index of the shorter axis */
};

/* Optimizer group reported by gpt_tensor_info. */
enum { GPT_GROUP_ADAMW = 0, GPT_GROUP_MUON = 1 };

/*
 * Model and batch configuration.
 *   depth     number of decoder blocks (the single shape knob)
 *   d_model   0 derives 64 * depth; any multiple of head_dim is accepted
 *   vocab     vocabulary size, a multiple of 8 (32768 in the pages' runs)
 *   batch     sequences per step; seq_len tokens each
 *   head_dim  must be 128; mlp_mult must be 4
 *   precision 0 = bf16 GEMMs; 1 = every GEMM of the attention output, MLP
 *             up and MLP down projections on fp8 e4m3 operands with dynamic
 *             per-tensor scales (448 / amax of the tensor, the amax kept by
 *             the kernel that produced it): the forward products X W, the
 *             activation gradients dY W^T and the weight gradients X^T dY,
 *             with X, W and dY quantised ("3. Gestión de Precisión": FP8
 *             with per-tensor scaling on most layers); the q|k|v projection
 *             (its rounding enters the QK-normalised attention logits),
 *             attention and the lm_head stay bf16
 *   ns_tf32_steps  operand precision of the five Newton-Schulz steps:
 *             -1 = fp16 operands at the full tensor rate, iterates carried as
 *             fp16 (high, low) pairs of about 22 significant bits
 *             (the recommended setting); 0..5 = that many leading steps with
 *             fp32 operands read as tf32 (half rate), the rest bf16.  fp16
 *             operands keep the update within ~1% of fp64 on the decaying
 *             spectra real gradients have, as three tf32 steps do; bf16-only
 *             steps amplify rounding on small singular values (up to ~8%).
 *   seed      seed of the N(0, 0.02) initial weights drawn by gpt_init
 */
typedef struct gpt_config {
  int32_t depth;
  int32_t d_model;
  int32_t vocab;
  int32_t batch;
  int32_t seq_len;
  int32_t head_dim;
  int32_t mlp_mult;
  int32_t precision;
  int32_t ns_tf32_steps;
  int32_t lm_chunk_rows; /* rows of logits held at once by the fused lm_head/CE; 0 = 8192 */
  uint64_t seed;
  int32_t short_window;   /* tokens of left context of an "S" layer (0 ..) */
  char window_pattern[12];/* per-layer attention window, repeated over the
                           * layers: 'S' = sliding window of short_window
                           * earlier tokens (query t sees keys t - short_window
                           * .. t), 'L' = full causal; e.g. "SSSL"; empty (all
                           * zero) = every layer full causal.  "¿Cómo Entrenar
                           * Tu Propio ChatGPT por $50?", section "1. Modelo
                           * GPT", sliding-window attention. */
  int32_t residual_extras;/* 1: the smear, per-layer residual and x0 scales
                           * and the backout of section "1. Modelo GPT"
                           * (efficiency tricks 1-3): the embedding e of
                           * position t becomes e[t] + smear sigmoid(w .
                           * e[t, :24]) e[t-1] (t > 0); before block i,
                           * x <- resid[i] x + x0s[i] x0 (x0 = the smeared
                           * embedding); after the last block,
                           * x <- x - backout * (stream entering block
                           * depth/2).  2*depth+26 scalars, tensor id
                           * 2 + 4*depth, trained by adamw_step, initialised
                           * to resid = 1 and everything else 0 (the plain
                           * network).  0: off. */
  int32_t ve_gate_channels; /* > 0: value embeddings of section "1. Modelo
                           * GPT" (value residual) on layers 0, 2, 4, ...:
                           * v[t, h] += 3 sigmoid(xn1[t, :C] . g[:, h])
                           * ve[tok[t], head h] with C = ve_gate_channels
                           * (at most min(d_model, 128), C * heads <= 1024),
                           * a [vocab, d] table and a [C, heads] gate per such
                           * layer, trained by adamw_step (tables N(0, 0.02),
                           * gates 0 at init).  0: off. */
  int32_t n_kv_head;      /* grouped kv heads (section "1. Modelo GPT", GQA):
                           * 0 = one per query head; else a divisor of the
                           * heads; the fused projection is then
                           * [d, d + 2 * 128 * n_kv_head] with columns
                           * q | k | v, query head h reading kv head
                           * h / (heads / n_kv_head); value-embedding tables
                           * and gates are per kv head. */
} gpt_config;

typedef struct gpt_ctx gpt_ctx;

/* Byte counts of the three caller-owned device buffers for cfg:
 *   param_bytes  fp32 masters and their bf16 working copies
 *   state_bytes  fp32 gradients, Muon momenta, AdamW moments
 *   act_bytes    saved activations, scratch and the small device scalars
 * Returns GPT_EINVAL for an unsupported configuration. */
int gpt_workspace_size(const gpt_config* cfg, size_t* param_bytes, size_t* state_bytes, size_t* act_bytes);

/* Binds the buffers and the CUDA stream (a cudaStream_t; NULL = legacy
 * default stream) to a new context.  Draws the initial weights on the
 * device (N(0, 0.02) rounded to bf16, masters equal to their bf16 copies:
 * the fp32 master weights of "Como Treinar Seu Próprio ChatGPT por 50
 * Dólares?", section "3. Gerenciamento de Precisão"), zeroes gradients and
 * optimizer state.  Synchronous. */
int gpt_init(const gpt_config* cfg, void* param_buf, void* state_buf, void* act_buf, void* stream,
             gpt_ctx** out);

/* Forward and backward pass over one batch of the decoder of "¿Cómo Entrenar
 * Tu Propio ChatGPT por $50?", section "1. Modelo GPT" (token embedding;
 * per block a gain-free RMSNorm, the fused q|k|v projection with rotary
 * embeddings and QK normalisation, causal attention, the output projection,
 * a second norm and the ReLU^2 MLP; a final norm, the untied lm_head and the
 * mean next-token cross-entropy), bf16 operands with fp32 accumulation
 * (section "3. Gestión de Precisión").
 *   tokens, targets  device int32 [batch, seq_len]; position t of a row
 *                    predicts targets[row, t] from tokens[row, 0..t]
 *   loss_out         device fp32 scalar, receives the mean cross-entropy
 *   accumulate       0: gradients are overwritten; 1: added to the stored ones
 * Ids outside [0, vocab) are treated as 0 and latched as GPT_ERANGE. */
int gpt_fwd_bwd(gpt_ctx* ctx, const int32_t* tokens, const int32_t* targets, float* loss_out, int accumulate);

/* Muon update ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2.
 * Optimizador Muon": momentum orthogonalised by five quintic Newton-Schulz
 * "Polar Express" steps) of every 2-D block matrix (fused q|k|v, attention
 * output, MLP up, MLP down; q|k|v is [d, 3d], narrower with grouped kv heads):
 * mom = momentum * mom + grad; X = NS5(mom / (||mom||_F + 1e-7))
 * with the Polar Express coefficients; W = W (1 - lr * weight_decay)
 * - lr * sqrt(max(1, rows / cols)) * X.  Refreshes the bf16 copies. */
int muon_step(gpt_ctx* ctx, float lr, float momentum, float weight_decay);

/* muon_step with the NorMuon variance reduction ("¿Cómo Entrenar Tu Propio
 * ChatGPT por $50?", section "2. Optimizador Muon", NorMuon snippet) applied
 * to each orthogonalised update X [rows, cols] before the weight update:
 *   v_mean = mean of X^2 over the longer axis (the columns when square), one
 *            value per index of the shorter axis (d values per matrix)
 *   V      = beta2 V + (1 - beta2) v_mean   (GPT_KIND_NORMUON_V; zero at init)
 *   s      = max(V, 1e-10)^(-1/2)
 *   X     <- X * s (along the shorter axis) * sqrt(sum v_mean)
 *            / max(sqrt(sum v_mean s^2), 1e-10)
 * so the update keeps its Frobenius norm.  beta2 outside [0, 1) is
 * GPT_EINVAL.  The page's snippet leaves the reduction axis and the second
 * norm undefined; the reading above is the one this library implements. */
int muon_step_normuon(gpt_ctx* ctx, float lr, float momentum, float weight_decay, float beta2);

/* Muon (normuon_beta2 < 0) or NorMuon (0 <= normuon_beta2 < 1, as
 * muon_step_normuon) of the block matrices of layers l0 .. l1-1 only, for
 * data-parallel ranks that split the optimizer work by layer: every matrix
 * is updated on its own, so the ranges of all ranks together give exactly
 * what one whole-model call gives.  The bf16 working copies of the updated
 * layers then have to reach the other ranks (gpt_block_region gives their
 * bytes).  0 <= l0 <= l1 <= depth, else GPT_EINVAL; l0 == l1 does nothing. */
int muon_step_layers(gpt_ctx* ctx, float lr, float momentum, float weight_decay, float normuon_beta2, int l0,
                     int l1);

/* Byte range of block matrix kind (0 fused q|k|v, 1 attention output, 2 MLP
 * up, 3 MLP down) for layers l0 .. l1-1: inside param_buf for
 * GPT_REGION_MASTER (fp32 masters) and GPT_REGION_BF16 (bf16 working
 * copies), inside state_buf for GPT_REGION_GRAD (fp32 gradients).  The
 * layers of one kind are contiguous, so the range is one span; the block
 * gradients follow those of the embedding and lm_head inside the
 * gpt_grad_region span. */
enum { GPT_REGION_MASTER = 0, GPT_REGION_BF16 = 1, GPT_REGION_GRAD = 2 };
int gpt_block_region(const gpt_ctx* ctx, int what, int kind, int l0, int l1, size_t* offset_bytes,
                     size_t* size_bytes);

/* AdamW update ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2.
 * Optimizador Muon", parameter table: embeddings and lm_head go to AdamW)
 * of the token embedding and lm_head (and of the residual-extras
 * scalars and value-embedding tables and gates when those are on) with bias
 * correction (the step count is kept in the context) and decoupled weight
 * decay. */
int adamw_step(gpt_ctx* ctx, float lr, float beta1, float beta2, float eps, float weight_decay);

/* adamw_step for data-parallel ranks that shard the AdamW state by rows
 * ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2. Optimizador
 * Muon", distributed training: ZeRO-2 sharding): only rows
 * [part R / nparts, (part + 1) R / nparts) of the token embedding (R = vocab)
 * and of the lm_head (R = d_model) are updated, with their moments and bf16
 * working copies; the residual-extras scalars and value-embedding tables and
 * gates, when on, are updated whole.  The step count advances by one, as for
 * adamw_step.  The parts of all ranks together give exactly what one
 * adamw_step gives; each rank then shares its rows' bf16 copies
 * (gpt_tensor_region).  0 <= part < nparts, else GPT_EINVAL. */
int adamw_step_shard(gpt_ctx* ctx, float lr, float beta1, float beta2, float eps, float weight_decay, int part,
                     int nparts);

/* The number of adamw_step calls so far (its bias correction uses it), for a
 * checkpoint: with every tensor's value and optimizer state (gpt_get_tensor)
 * it restores a context exactly.  A negative count is GPT_EINVAL. */
int gpt_get_adam_step(const gpt_ctx* ctx, int64_t* step);
int gpt_set_adam_step(gpt_ctx* ctx, int64_t step);

/* Whole step from HOST buffers: copies tokens and targets (int32
 * [batch, seq_len], pinned memory recommended) to the device, runs
 * gpt_fwd_bwd, muon_step and adamw_step with the given hyper-parameters,
 * copies the loss back to *loss_host and synchronises the stream. */
typedef struct gpt_hparams {
  float muon_lr, muon_momentum, muon_wd;
  float adam_lr, adam_beta1, adam_beta2, adam_eps, adam_wd;
} gpt_hparams;
int gpt_train_step_host(gpt_ctx* ctx, const int32_t* tokens_host, const int32_t* targets_host,
                        const gpt_hparams* hp, float* loss_host);

/* Parameter tensors: id 0 = token embedding [vocab, d], 1 = lm_head [d, vocab],
 * 2 + 4 l + j for block l with j = 0 fused q|k|v [d, 3d] (d + 256 n_kv_head
 * columns with grouped kv heads), 1 attention output
 * [d, d], 2 MLP up [d, 4d], 3 MLP down [4d, d]; with residual_extras, id
 * 2 + 4 depth = the scalars [1, 2 depth + 26] (resid[0..depth),
 * x0s[0..depth), backout, smear, smear gate weights[24]); with value
 * embeddings, the next ceil(depth / 2) ids are their tables [vocab, d] (layers
 * 0, 2, ...) and the one after them all gates [n * C, heads] (layer 2i's
 * gate in rows i*C .. i*C+C-1). */
int gpt_num_tensors(const gpt_ctx* ctx);
int gpt_tensor_info(const gpt_ctx* ctx, int id, int32_t* rows, int32_t* cols, int32_t* group);

/* Device-to-device copies of rows*cols fp32 values (asynchronous); d values
 * for GPT_KIND_NORMUON_V. */
int gpt_get_tensor(gpt_ctx* ctx, int id, int kind, float* dst);
int gpt_set_tensor(gpt_ctx* ctx, int id, int kind, const float* src);

/* Byte range of rows row0 .. row1-1 of tensor id (the embedding, the lm_head
 * or a block matrix; ids as for gpt_tensor_info) inside param_buf for
 * GPT_REGION_MASTER (fp32) and GPT_REGION_BF16 (the bf16 working copy), or
 * inside state_buf for GPT_REGION_GRAD (fp32 gradient).  Rows are contiguous
 * (row-major), so the range is one span.  Other ids, or a row range outside
 * [0, rows], are GPT_EINVAL. */
int gpt_tensor_region(const gpt_ctx* ctx, int what, int id, int row0, int row1, size_t* offset_bytes,
                      size_t* size_bytes);

/* Gradient buckets, in the order in which gpt_fwd_bwd completes them: 0 the
 * lm_head (done once the last lm_head chunk is through, early in the
 * backward), 1..4 one block matrix kind over every layer (fused q|k|v,
 * attention output, MLP up, MLP down; each done by one batched
 * weight-gradient launch after the backward sweep), 5 the token embedding
 * with the residual-extras and value-embedding gradients (done at the end).
 * Each bucket is one span of state_buf (gpt_grad_bucket); together they tile
 * the gpt_grad_region span, which is laid out in this order. */
enum { GPT_GRAD_BUCKETS = 6 };
int gpt_grad_bucket(const gpt_ctx* ctx, int bucket, size_t* offset_bytes, size_t* size_bytes);

/* Registers n <= GPT_GRAD_BUCKETS caller-owned CUDA events (cudaEvent_t,
 * created by the caller on the context's device): every later gpt_fwd_bwd
 * records events[i] on the context's stream as soon as bucket i is complete,
 * so a data-parallel caller can start reducing a bucket on another stream
 * (cudaStreamWaitEvent) while the backward still runs.  n = 0 stops the
 * recording.  The events must outlive their registration. */
int gpt_set_grad_events(gpt_ctx* ctx, void* const* events, int n);

/* Byte range of the fp32 gradients of every parameter inside state_buf
 * (one contiguous span; alignment padding inside it stays zero).  Data
 * parallel training averages this span across ranks between gpt_fwd_bwd and
 * the optimizer calls. */
int gpt_grad_region(const gpt_ctx* ctx, size_t* offset_bytes, size_t* size_bytes);

/* Per-position cross-entropy of the last gpt_fwd_bwd: batch * seq_len fp32
 * values (row-major [batch, seq_len]) copied device-to-device into dst. */
int gpt_get_row_loss(gpt_ctx* ctx, float* dst);

/* Launch-site categories for the event profiler. */
enum {
  GPT_PROF_QKV_GEMM = 0,  /* q|k|v projection + RoPE + QK-norm epilogue */
  GPT_PROF_PROJ_GEMM,     /* attention output projection + residual add */
  GPT_PROF_FC_GEMM,       /* MLP up projection + ReLU^2 */
  GPT_PROF_DOWN_GEMM,     /* MLP down projection + residual add */
  GPT_PROF_ATTN_FWD,      /* causal flash attention forward */
  GPT_PROF_ATTN_BWD,      /* causal flash attention backward (with its D pre-pass) */
  GPT_PROF_LOGITS_GEMM,   /* lm_head logits + per-tile softmax partials */
  GPT_PROF_CE_FINISH,     /* log-sum-exp, row loss, dlogits in place */
  GPT_PROF_LM_DX_GEMM,    /* dlogits W_lm^T (+ split-K reduce) */
  GPT_PROF_LM_DW_GEMM,    /* xf^T dlogits */
  GPT_PROF_DX_GEMM,       /* block activation-gradient GEMMs */
  GPT_PROF_DW_GEMM,       /* block weight-gradient GEMMs (+ split-K reduce) */
  GPT_PROF_NORM,          /* RMSNorm forward and backward */
  GPT_PROF_QK_BWD,        /* QK-norm and RoPE backward */
  GPT_PROF_EMBED,         /* embedding forward and backward, id checks */
  GPT_PROF_NS_GEMM,       /* Newton-Schulz GEMMs */
  GPT_PROF_MUON_ELEM,     /* Muon momentum, norms, normalise, apply */
  GPT_PROF_ADAMW,         /* AdamW */
  GPT_PROF_FP8_QUANT,     /* fp8 amax and e4m3 quantisation (precision 1) */
  GPT_PROF_COUNT
};

/* Record CUDA events around every launch of the categories set in mask
 * (bit i = category i); 0 turns recording off. */
int gpt_profile_enable(gpt_ctx* ctx, uint32_t mask);

/* Synchronises the stream, then writes per category the summed device time
 * (ms) and the number of recorded launches since the last read (arrays of
 * GPT_PROF_COUNT entries; either may be NULL), and clears the record. */
int gpt_profile_read(gpt_ctx* ctx, double* ms, int64_t* launches);

/* Synchronises the stream and reports (then clears) latched device errors. */
int gpt_check(gpt_ctx* ctx);

/* Bound of every device-side wait of this context's kernels, in SM clock
 * cycles (the waits of the TMA / tensor-core / softmax pipelines inside the
 * GEMM and attention kernels); cycles <= 0 restores the default of 4e9
 * (about 2 s at 2 GHz).  When a wait runs past its bound the kernel stops,
 * lets its in-flight copies land, frees its tensor memory and returns;
 * gpt_check then reports GPT_ETIMEOUT and the step's results are invalid,
 * but the context stays usable.  A short bound is for failure-detection
 * tests only: it makes ordinary waits expire. */
int gpt_set_wait_limit(gpt_ctx* ctx, long long cycles);

/* Number of kernels the library has launched through this context. */
int64_t gpt_launch_count(const gpt_ctx* ctx);

void gpt_destroy(gpt_ctx* ctx);
const char* gpt_last_error(void);

/* --------------------------------------------------------------------
 * Op-level entry points: single kernels of the step on caller buffers,
 * for testing and for composing other models.  All pointers are device
 * pointers; the stream is a cudaStream_t; asynchronous.  The return code
 * covers argument checks and the launch; failures inside the kernels (an
 * expired bounded wait) are latched in a device error word that the
 * library keeps for each GPU and reported by gpt_op_check.
 * ------------------------------------------------------------------ */

/* Synchronises the stream, then reports and clears the op-level error word
 * of the current device: GPT_ETIMEOUT if a bounded device wait of an
 * op-level call expired since the last check (that call's outputs are
 * invalid), GPT_OK otherwise.  The word is shared by every op-level call on
 * the device, whatever its stream or thread. */
int gpt_op_check(void* stream);

/* Bound of the device-side waits of every later op-level call in this
 * process, in SM clock cycles; cycles <= 0 restores the default (4e9).  As
 * for gpt_set_wait_limit, a short bound is for failure-detection tests. */
int gpt_op_set_wait_limit(long long cycles);

/* C[z] = A[z] * B[z] with fp32 accumulation on the tensor cores.
 *   A [M, K] row-major bf16 (z stride M*K), B [K, N] row-major bf16 (z stride K*N),
 *   C [M, N] row-major fp32 (z stride M*N).  N and K multiples of 8.
 *   a_trans / b_trans = 1 read A as [K, M] and B as [N, K] instead. */
int gpt_op_matmul_bf16(const void* A, const void* B, float* C, int M, int N, int K, int batch, int a_trans,
                       int b_trans, void* stream);

/* C = A * B^T with fp32 operands read as tf32 by the tensor cores
 * (kind::tf32), fp32 accumulation.  A [M, K] row-major fp32, B given as
 * [N, K] row-major fp32 (b_trans must be 1: both operands are staged
 * K-major), C [M, N] fp32.  K a multiple of 4, N of 8.  b_trans = 0 is
 * GPT_EINVAL. */
int gpt_op_matmul_tf32(const float* A, const float* B, float* C, int M, int N, int K, int b_trans, void* stream);

/* Per-tensor e4m3 quantisation ("3. Gestión de Precisión": FP8 training with
 * per-tensor scaling): q = e4m3(x * 448 / amax|x|), round to nearest even,
 * saturating at +-448; *inv = amax / 448 (1 if x is all zero).
 *   x: n bf16 values (16-byte aligned); q: n bytes (8-byte aligned);
 *   amax_scratch: one device word. */
int gpt_op_quantize_e4m3(const void* x, long long n, void* q, float* inv, unsigned int* amax_scratch, void* stream);

/* C = (A * B) * inv_a * inv_b on e4m3 operands (tcgen05 kind::f8f6f4), fp32
 * accumulation.  A [M, K] row-major bytes; B [K, N] row-major, or [N, K] with
 * b_trans = 1; inv_a, inv_b: device inverse scales; C [M, N] fp32.
 * N and K multiples of 16. */
int gpt_op_matmul_fp8(const void* A, const void* B, float* C, int M, int N, int K, const float* inv_a,
                      const float* inv_b, int b_trans, void* stream);

/* Causal attention forward: q, k, v bf16 [B, H, T, 128] -> o bf16 [B, T, H, 128]
 * and lse fp32 [B, H, T] (natural log of the softmax denominator of
 * q.k / sqrt(128)). */
int gpt_op_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int T,
                         void* stream);

/* Causal attention backward: given o, lse from the forward and dout bf16
 * [B, T, H, 128], writes dq fp32, dk and dv bf16 [B, H, T, 128]; Dscratch is
 * fp32 [B, H, T]. */
int gpt_op_attention_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, float* Dscratch, float* dq, void* dk, void* dv, int B, int H, int T,
                         void* stream);

/* The two attention variants of "¿Cómo Entrenar Tu Propio ChatGPT por $50?",
 * section "1. Modelo GPT": grouped kv heads (GQA) and sliding-window
 * attention.  q bf16 [B, H, T, 128]; k, v bf16 [B, Hkv, T, 128] with Hkv
 * dividing H, query head h reading kv head h / (H / Hkv); window < 0 (or
 * >= T) is full causal attention, else query t sees keys t - window .. t.
 * Forward outputs as gpt_op_attention_fwd; the backward writes dq fp32
 * [B, H, T, 128] and dk, dv bf16 [B, Hkv, T, 128], each the sum over the
 * query heads of its group.  A bad head split is GPT_EINVAL. */
int gpt_op_attention_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                            int T, int window, void* stream);
int gpt_op_attention_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dout,
                            const float* lse, float* Dscratch, float* dq, void* dk, void* dv, int B, int H, int Hkv,
                            int T, int window, void* stream);

/* Embedding gradient ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section
 * "1. Modelo GPT": the token embedding x0 = wte[tok]; its gradient scatters
 * the rows of dx by token): dwte[v] (+)= sum of dx[m] over the positions m
 * with tokens[m] = v, summed in position order (deterministic, whatever the
 * token histogram).
 *   tokens  device int32 [M]; ids outside [0, vocab) count as 0
 *   dx      fp32 [M, d]; dwte fp32 [vocab, d] (zeroed first unless
 *           accumulate); d a multiple of 128, both 16-byte aligned
 *   scratch device buffer of gpt_op_embedding_bwd_scratch(M, d) bytes,
 *           256-byte aligned (0 for a bad shape) */
size_t gpt_op_embedding_bwd_scratch(int M, int d);
int gpt_op_embedding_bwd(const int32_t* tokens, const float* dx, float* dwte, int M, int d, int vocab, int accumulate,
                         void* scratch, void* stream);

/* Gain-free RMSNorm of fp32 rows [M, d] -> bf16 y and fp32 rstd [M]. */
int gpt_op_rmsnorm_fwd(const float* x, void* y, float* rstd, int M, int d, void* stream);

/* Newton-Schulz ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2.
 * Optimizador Muon": Polar Express, five steps) of a batch of fp32 matrices
 * G [batch, rows, cols] -> fp32 X of the same shape, via the same kernels
 * as muon_step; tf32_steps selects the operand precision as ns_tf32_steps
 * does (-1 = fp16 operands, 0..5 = leading tf32 steps then bf16); scratch
 * is a device buffer of gpt_op_newton_schulz_scratch() bytes. */
size_t gpt_op_newton_schulz_scratch(int batch, int rows, int cols);
int gpt_op_newton_schulz(const float* G, float* X, int batch, int rows, int cols, int tf32_steps, void* scratch,
                         void* stream);

/* Newton-Schulz without any device allocation (the pages have no
 * counterpart of this call).  Same computation and arguments as
 * gpt_op_newton_schulz, but its scratch is a fixed array in device memory
 * that belongs to the loaded library, for callers that cannot hand device
 * scratch to the library: code whose device memory is owned entirely by
 * another allocator, runtimes that forbid cudaMalloc after start-up, and
 * interfaces with no place for a scratch pointer.
 *   Limits: batch * rows * cols <= 262144 fp32 elements and batch <= 64;
 *   larger inputs return GPT_EINVAL.  The array (6,832,384 bytes) stays
 *   resident on every GPU that loads the library until the process exits.
 *   Every call looks up the array's device address with the current device
 *   (so after a device reset the new context's address is used); the first
 *   lookup on a device loads the library's device code there, so make the
 *   first call on each device before any stream capture.  Expired device
 *   waits are reported by gpt_op_check.
 *   All calls share the one array: calls that overlap on the GPU (other
 *   streams, other threads) race on it and must be serialised by the caller.
 * This call performs no cudaMalloc/cudaFree and calls no allocating
 * library routine. */
int gpt_op_newton_schulz_noalloc(const float* G, float* X, int batch, int rows, int cols, int tf32_steps,
                                 void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPT_B200_H */

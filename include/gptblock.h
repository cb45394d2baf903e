/* gptblock.h — C ABI of the B200 (sm_100a) GPT block library.
 *
 * One training step (forward + backward) of the nanochat GPT transformer
 * block stack, as described on the source pages:
 *   apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour 50€ ?",
 *   § "Comment nanochat fonctionne" › 1. Le modèle GPT (feature list: RoPE,
 *   QK normalisation, untied embedding / output projection, ReLU², GQA,
 *   sliding-window attention; value-embedding snippet; "efficiency tricks"
 *   snippets: per-layer residual lambdas, smear, backout) and § 3 "Gestion de
 *   la précision" (Linear casts the weight to the activation dtype; FP8 with
 *   per-tensor scaling).
 *
 * Conventions for every entry point
 *   - Every tensor pointer is a DEVICE pointer allocated by the caller (for
 *     example through PyTorch).  The library never allocates or frees device
 *     memory; buffers it needs beyond inputs and outputs come from a
 *     caller-owned workspace whose size gptb_workspace_bytes() reports.
 *   - Activations are row-major and token-major: [B, T, features].  Weights
 *     follow nn.Linear, [out, in], and every projection is y = x W^T.
 *   - Storage dtype (cfg.dtype): GPTB_F32 -> float; GPTB_BF16 and
 *     GPTB_FP8_E4M3 -> bf16 storage (FP8 only changes the GEMM operands).
 *   - Scalars (lambdas) are fp32 device values.  All gradients are fp32 and
 *     ACCUMULATED (+=); the caller zeroes them before the first micro-step,
 *     which makes gradient accumulation free.
 *   - All work is enqueued on `stream`; no call synchronises the host except
 *     gptb_device_error().  Pointers must be 16-byte aligned.
 *   - Return value: GPTB_OK (0) or a negative GPTB_ERR_* code; nothing is
 *     enqueued when an argument check fails.  No exceptions cross the ABI.
 */
#ifndef GPTBLOCK_H
#define GPTBLOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gptb_stream_t; /* same type as cudaStream_t */

enum {
  GPTB_OK = 0,
  GPTB_ERR_INVALID_ARG = -1, /* null / misaligned pointer, inconsistent shape */
  GPTB_ERR_UNSUPPORTED = -2, /* dtype, head_dim or device not supported      */
  GPTB_ERR_CUDA = -3,        /* a CUDA call or kernel launch failed          */
  GPTB_ERR_TIMEOUT = -4,     /* a bounded device wait expired (see below)    */
  GPTB_ERR_WORKSPACE = -5,   /* workspace too small                          */
  GPTB_ERR_BAD_INPUT = -6    /* a device-side check found invalid input data
                                (a target id outside [0, vocab)); reported by
                                gptb_device_error()                          */
};

enum { GPTB_F32 = 0, GPTB_BF16 = 1, GPTB_FP8_E4M3 = 2 };

#define GPTB_MAX_LAYERS 64

/* Model shape and options.  Plain data, passed by pointer, copied by callee. */
typedef struct {
  int B, T;            /* batch rows, tokens per row                              */
  int d;               /* model width, multiple of 8, <= 2048                     */
  int n_head;          /* query heads H                                           */
  int n_kv_head;       /* key/value heads Hkv, H % Hkv == 0 (GQA)                 */
  int head_dim;        /* hd: 128 for bf16/fp8; <= 128 and even for f32           */
  int mlp_hidden;      /* F (4*d in nanochat), multiple of 8                      */
  int vocab;           /* V, multiple of 8                                        */
  int n_layer;         /* L <= GPTB_MAX_LAYERS                                    */
  int window[GPTB_MAX_LAYERS]; /* per layer: -1 full causal, else W: keys t-W..t  */
  int has_ve[GPTB_MAX_LAYERS]; /* per layer: 1 = gated value embedding            */
  int ve_gate_ch;      /* channels feeding the VE gate (32)                       */
  int smear_ch;        /* channels feeding the smear gate (24); 0 = smear off     */
  int backout_layer;   /* layer whose input is subtracted after the last; -1 off  */
  float rope_base;     /* 10000                                                   */
  float norm_eps;      /* RMSNorm epsilon inside the rsqrt (1e-6)                 */
  int dtype;           /* GPTB_F32 | GPTB_BF16 | GPTB_FP8_E4M3                    */
  int fp8_flags;       /* GPTB_FP8_E4M3 configs only (0 otherwise), bits:
                          GPTB_FP8_GRAD_E5M2: gradient operands of the input- and
                            weight-gradient GEMMs in e5m2 (scale 57344/amax);
                          GPTB_FP8_LM_HEAD: the lm_head GEMMs in FP8 too (logits
                            from e4m3 hf and W_lm; the logits gradient, whose
                            entries lie in [-1/N, 1/N], with the fixed scale
                            qmax*N, in e5m2 with GPTB_FP8_GRAD_E5M2)          */
} gptb_config;

enum { GPTB_FP8_GRAD_E5M2 = 1, GPTB_FP8_LM_HEAD = 2 };

/* Weights of one block (storage dtype).  w_ve_gate / ve_table only on
 * value-embedding layers (NULL elsewhere). */
typedef struct {
  const void* w_qkv;      /* [(H+2Hkv)*hd, d]: rows q heads, then k, then v     */
  const void* w_o;        /* [d, H*hd]                                          */
  const void* w_fc;       /* [F, d]                                             */
  const void* w_proj;     /* [d, F]                                             */
  const void* w_ve_gate;  /* [Hkv, ve_gate_ch]                                  */
  const void* ve_table;   /* [V, Hkv*hd]                                        */
  const float* lambdas;   /* device fp32 [2]: resid_lambda, x0_lambda           */
} gptb_block_weights;

/* Gradients of one block, fp32, accumulated (+=), same shapes as above. */
typedef struct {
  float* w_qkv;
  float* w_o;
  float* w_fc;
  float* w_proj;
  float* w_ve_gate;  /* may be NULL on layers without VE                         */
  float* ve_table;   /* dense [V, Hkv*hd] scatter-add target; NULL without VE    */
  float* lambdas;    /* [2]                                                      */
} gptb_block_grads;

typedef struct {
  const void* wte;           /* [V, d] token embedding                         */
  const void* w_lm;          /* [V, d] untied output projection                */
  const void* w_smear_gate;  /* [smear_ch]                                     */
  const float* smear_lambda; /* device fp32 scalar                             */
  const float* backout_lambda; /* device fp32 scalar                           */
  gptb_block_weights layers[GPTB_MAX_LAYERS];
} gptb_model_weights;

typedef struct {
  float* wte;
  float* w_lm;
  float* w_smear_gate;
  float* smear_lambda;
  float* backout_lambda;
  gptb_block_grads layers[GPTB_MAX_LAYERS];
} gptb_model_grads;

/* Workspace kinds for gptb_workspace_bytes(). */
enum {
  GPTB_WS_BLOCK_SAVED = 0,   /* activations one block saves for its backward    */
  GPTB_WS_BLOCK_SCRATCH = 1, /* temporaries of one block forward/backward        */
  GPTB_WS_LM_HEAD = 2,       /* temporaries of lm_head_xent                      */
  GPTB_WS_STACK = 3          /* everything gpt_stack_step needs                  */
};

/* Bytes of workspace of the given kind for this config (0 on a bad config). */
size_t gptb_workspace_bytes(const gptb_config* cfg, int kind);

/* One block forward (layer `layer` of cfg; its window / has_ve apply).
 *   x, x0  [B,T,d]  block input and the stack's x0 (the smeared embedding)
 *   idx    [B,T] int32 token ids (value-embedding lookup)
 *   x_out  [B,T,d]  block output
 *   saved  GPTB_WS_BLOCK_SAVED bytes, filled here, read by the backward
 *   scratch GPTB_WS_BLOCK_SCRATCH bytes
 * Computes xm = a x + b x0; h = rmsnorm(xm); q,k,v = h Wqkv^T;
 * v += 3 sigmoid(h[:, :C] Wg^T) VE[idx]; q,k = rope(rmsnorm_per_head(q,k));
 * x1 = xm + attn(q,k,v) Wo^T; x_out = x1 + relu(rmsnorm(x1) Wfc^T)^2 Wproj^T. */
int gpt_block_forward(const gptb_config* cfg, int layer, const gptb_block_weights* w, const void* x,
                      const void* x0, const int32_t* idx, void* x_out, void* saved, void* scratch,
                      gptb_stream_t stream);

/* One block backward from dL/dx_out.  Needs the forward's x, x0, idx and
 * saved buffer.  Writes dx [B,T,d] (storage dtype), ACCUMULATES dx0_accum
 * [B,T,d] (fp32) and every gradient in g.  dx_extra (nullable, storage dtype)
 * is added to dx (used for the backout term). */
int gpt_block_backward(const gptb_config* cfg, int layer, const gptb_block_weights* w, const void* x,
                       const void* x0, const int32_t* idx, const void* saved, const void* dx_out,
                       const void* dx_extra, void* dx, float* dx0_accum, gptb_block_grads* g, void* scratch,
                       gptb_stream_t stream);

/* Untied lm_head + mean next-token cross-entropy over N = B*T rows without
 * materialising the full [N, V] logits (row chunks of at most 8192 tokens).
 * Source: the same page, § 1 feature list (untied embedding and output
 * projection); dev.to/aakira "ChatGPTを50ドルでトレーニングする方法", table of
 * what nanochat covers (BPE vocabulary 32,768).
 *   h [N,d] (normed final hidden state), w_lm [V,d], targets [N] int32
 *   loss_out: device fp32 scalar (written, the mean over N)
 *   dh [N,d] storage dtype (written); dw_lm [V,d] fp32 (accumulated)
 *   ws: GPTB_WS_LM_HEAD bytes.
 * bf16 and FP8 configs (the lm_head stays bf16 in FP8 configs): the logits
 * GEMM's epilogue emits each row's softmax statistics per 256-column tile and
 * z at the target, a warp per row combines them into the log-sum-exp, and one
 * streaming pass writes the gradient (softmax - onehot)/N over the chunk's
 * logits, which the dh and dW GEMMs read.  fp32 configs: SIMT GEMMs and a
 * two-pass row kernel.
 * targets must lie in [0, vocab).  A target outside that range is never read
 * as an index: its row's loss term is 0 and its gradient lacks the one-hot
 * term, and gptb_device_error() returns GPTB_ERR_BAD_INPUT afterwards (the
 * call's results are then not meaningful). */
int lm_head_xent(const gptb_config* cfg, const void* h, const void* w_lm, const int32_t* targets, float* loss_out,
                 void* dh, float* dw_lm, void* ws, gptb_stream_t stream);

/* (GPTB_FP8_LM_HEAD configs: lm_head_xent_noalloc returns GPTB_ERR_UNSUPPORTED,
 * since the FP8 copies of hf and W_lm need the workspace.) */

/* lm_head_xent without a workspace, for callers that cannot allocate device
 * memory themselves: for example a plugin or C caller that is handed tensors
 * and a stream by a host framework whose allocator owns all device memory, or
 * a latency-critical path that must not call cudaMalloc (which can
 * synchronise the device).  No counterpart on the source pages: this is a
 * convenience of this library.
 *   Same arguments, results, target rule and accumulation (+= into dw_lm) as
 *   lm_head_xent, minus `ws`.  Its scratch is one file-scope device array of
 *   8 MiB of logits, 1 MiB of per-tile softmax statistics and 768 KiB of
 *   per-row values (losses, z at the target, log-sum-exp), held by every GPU
 *   that loads the library until the process exits.  Limits: B*T <= 65536
 *   and vocab * element size <= 8 MiB (otherwise GPTB_ERR_WORKSPACE, nothing
 *   enqueued).  Rows are processed in chunks of
 *   min(8 MiB / (vocab * element size), 1 MiB / (8 * ceil(vocab / 256)))
 *   rows (128 rows for vocab 32768 in bf16).
 *   Every call looks up the array's device address on the current device;
 *   the first call on a device also loads the library's kernels there, so
 *   make that first call before any stream capture.  Nothing is allocated or
 *   freed.  All calls share the one array and every call overwrites it:
 *   calls that overlap on the GPU (other streams, other threads) race and
 *   give wrong results; serialise them. */
int lm_head_xent_noalloc(const gptb_config* cfg, const void* h, const void* w_lm, const int32_t* targets,
                         float* loss_out, void* dh, float* dw_lm, gptb_stream_t stream);

/* Whole training step of the stack: embed -> smear -> L blocks -> backout ->
 * final RMSNorm -> lm_head + cross-entropy, then the full backward.  Writes
 * loss_out (device fp32 scalar) and accumulates every gradient in g.
 * ws: GPTB_WS_STACK bytes.  bf16/fp8 configs (lm_head present). */
int gpt_stack_step(const gptb_config* cfg, const gptb_model_weights* w, const int32_t* idx, const int32_t* targets,
                   float* loss_out, gptb_model_grads* g, void* ws, gptb_stream_t stream);

/* gpt_stack_step for data-parallel training: identical work, plus a host
 * callback ready(layer, user) made on the calling thread while the step is
 * being enqueued, right after the last kernel that writes block `layer`'s
 * weight gradients has been put on `stream` (layers in backward order,
 * L-1 down to 0), and once more with layer = -1 after the embedding / smear /
 * backout / lm_head gradients.  Work the callback enqueues on `stream`, or on
 * another stream after an event recorded on `stream`, runs once those
 * gradients are complete: the caller launches that layer's gradient
 * reduction there, overlapping the rest of the backward (the ZeRO-2 phase 1
 * of the page's "Entraînement distribué" section, bucketed per layer).  The
 * callback must not call back into this library.  No counterpart on the
 * pages beyond that section. */
typedef void (*gptb_grads_ready_fn)(int layer, void* user);
int gpt_stack_step_hooked(const gptb_config* cfg, const gptb_model_weights* w, const int32_t* idx,
                          const int32_t* targets, float* loss_out, gptb_model_grads* g, void* ws, gptb_stream_t stream,
                          gptb_grads_ready_fn ready, void* user);

/* Plain GEMM entry point used by the tests of the tensor-core kernel:
 * C[M,N] (+)= A[M,K] B[N,K]^T (bf16 operands, fp32 accumulate).
 *   a_mn / b_mn: 0 = operand stored K-major (row-major [M,K] / [N,K]),
 *                1 = stored MN-major (row-major [K,M] / [K,N]);
 *   lda, ldb: row strides in elements of the stored matrices;
 *   c_f32: 1 -> C is float and ACCUMULATED (+=, split-K allowed),
 *          0 -> C is bf16 and overwritten; ldc in elements. */
int gptb_gemm_bf16(const void* A, int a_mn, long long lda, const void* B, int b_mn, long long ldb, void* C,
                   int c_f32, long long ldc, int M, int N, int K, gptb_stream_t stream);

/* Batched form of gptb_gemm_bf16: for b = 0..batch-1, the matrices starting
 * b*stride_a, b*stride_b, b*stride_c elements after A, B, C (strides in
 * elements; their byte sizes multiples of 16) are multiplied as above, all in
 * one launch (the form the Polar Express products take over same-shape
 * matrices).  GPTB_ERR_INVALID_ARG for batch < 1 or a misaligned stride. */
int gptb_gemm_bf16_batched(const void* A, int a_mn, long long lda, long long stride_a, const void* B, int b_mn,
                           long long ldb, long long stride_b, void* C, int c_f32, long long ldc, long long stride_c,
                           int M, int N, int K, int batch, gptb_stream_t stream);

/* FP8 GEMM entry point used by the tests of the e4m3 / e5m2 tensor-core path:
 * C[M,N] += dequant(q(A) q(B)^T), fp32 accumulate, where q casts the bf16
 * operand to FP8 per tensor (A: e4m3 with scale 448/amax, or e5m2 with
 * 57344/amax when a_e5m2; B: e4m3), RNE, saturating.  Layout flags as in
 * gptb_gemm_bf16 (a_mn = 1 with b_mn = 0 is not supported); the operands must
 * be dense (lda, ldb = their inner extents, multiples of 16).  workspace:
 * device, gptb_gemm_fp8_workspace_bytes(M, N, K) bytes, 256-byte aligned. */
size_t gptb_gemm_fp8_workspace_bytes(int M, int N, int K);
int gptb_gemm_fp8(const void* A, int a_mn, long long lda, const void* B, int b_mn, long long ldb, float* C,
                  long long ldc, int M, int N, int K, int a_e5m2, void* workspace, size_t workspace_bytes,
                  gptb_stream_t stream);

/* ---------------------------------------------------- optimizer step ----
 * The step after the training step (nanochat's mixed optimizer: AdamW for the
 * embeddings, the lm_head and the scalar parameters; Muon, whose update is
 * orthogonalised by the Polar Express iteration, for the 2-D matrices).
 * Source: apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour 50€ ?",
 * § "Comment nanochat fonctionne" › 2 "L'optimiseur Muon"; dev.to/aakira
 * "ChatGPTを50ドルでトレーニングする方法" § 2 (parameter groups). */

/* One AdamW step over n fp32 parameters, in place:
 *   m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;
 *   p = p (1 - lr wd) - lr (m / (1-b1^step)) / (sqrt(v / (1-b2^step)) + eps).
 * p, m, v: device fp32 [n], updated; g: device fp32 [n], read.  p_bf16:
 * device bf16 [n] that receives the new p rounded to nearest-even (the
 * working copy the GEMMs read), or NULL.  step >= 1.  Errors:
 * GPTB_ERR_INVALID_ARG for null arrays, n < 0 or step < 1 (nothing enqueued). */
int gptb_adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, long long n, float lr, float beta1,
                    float beta2, float eps, float weight_decay, int step, gptb_stream_t stream);

/* Device workspace in bytes of gptb_polar_express for an [m, n] matrix. */
size_t gptb_polar_express_workspace_bytes(int m, int n, int steps);

/* Polar Express orthogonalisation of a 2-D update G [m, n] (bf16, row-major,
 * row stride n) into out [m, n] (bf16; must not overlap G): X = G / ||G||_F,
 * then for each (a, b, c) of coeffs[0..steps-1]:
 *   A = X^T X,  B = b A + c A A,  X = a X + X B
 * with A the Gram matrix of the smaller side (a wide G runs the same loop on
 * G^T, written back untransposed).  Every product is a tensor-core GEMM with
 * bf16 operands and fp32 accumulation; A, B and X are stored in bf16.
 * coeffs: HOST float [3*steps] (a, b, c per step; copied before return).
 * workspace: device, gptb_polar_express_workspace_bytes(m, n, steps) bytes.
 * Errors: GPTB_ERR_INVALID_ARG (m or n not a positive multiple of 8, steps
 * < 1 or > 64, null pointers), GPTB_ERR_WORKSPACE (too small),
 * GPTB_ERR_UNSUPPORTED (not an sm_100 device). */
int gptb_polar_express(const void* G, void* out, int m, int n, const float* coeffs, int steps, void* workspace,
                       size_t workspace_bytes, gptb_stream_t stream);

/* Device workspace in bytes of gptb_muon_step for an [m, n] matrix. */
size_t gptb_muon_workspace_bytes(int m, int n, int steps);

/* One Muon step on a 2-D weight W [m, n] (rows = output neurons), in place.
 * Sources: the same page, § 2 (the Polar Express loop, two of its five
 * coefficient tuples, the NorMuon lines); K. Jordan et al., "Muon: An
 * optimizer for hidden layers in neural networks" (2024) for the Nesterov
 * momentum; N. Amsel et al., "The Polar Express" (2025) for the five tuples;
 * Z. Li et al., "NorMuon" (2025) for the per-neuron second moment.
 *   buf = mu buf + g;  u = g + mu buf                       (momentum, Nesterov)
 *   o = Polar Express of u over coeffs[0..steps-1]          (as gptb_polar_express)
 *   v = beta2 v + (1-beta2) mean_row(o^2);  step = 1/sqrt(max(v, 1e-10))
 *   scale_row = step_row * sqrt(sum mean_row(o^2)) / max(sqrt(sum mean_row(o^2) step_row^2), 1e-10)
 *   w = w (1 - lr wd) - lr o scale_row;  w_bf16 = bf16(w)   (the update keeps the norm of o)
 * w: device fp32 [m, n] (updated); w_bf16: device bf16 [m, n] receiving the
 * new weight rounded to nearest-even, or NULL; g: device fp32 [m, n] (read);
 * buf: device fp32 [m, n] momentum (updated); v: device fp32 [m] second
 * moment (updated).  coeffs: HOST float [3*steps].  workspace: device,
 * gptb_muon_workspace_bytes(m, n, steps) bytes, 256-byte aligned.  Errors:
 * GPTB_ERR_INVALID_ARG (m or n not a positive multiple of 8, steps outside
 * 1..64, null or misaligned pointers), GPTB_ERR_WORKSPACE, GPTB_ERR_UNSUPPORTED
 * (not an sm_100 device). */
int gptb_muon_step(float* w, void* w_bf16, const float* g, float* buf, float* v, int m, int n, const float* coeffs,
                   int steps, float lr, float mu, float beta2, float weight_decay, void* workspace,
                   size_t workspace_bytes, gptb_stream_t stream);

/* gptb_muon_step on `count` (1..64) matrices of the same shape [m, n] at
 * once: every Polar Express product runs as one batched GEMM over the count
 * matrices (one launch instead of count, and count times the tiles to spread
 * over the SMs).  w, w_bf16, g, buf, v: HOST arrays of count device pointers,
 * each as in gptb_muon_step (w_bf16 may be NULL, or hold NULL entries); the
 * result for each matrix is that of gptb_muon_step up to the order of float
 * additions in the two NorMuon sums and the Frobenius norm.  workspace:
 * device, gptb_muon_batched_workspace_bytes(count, m, n, steps) bytes,
 * 256-byte aligned.  Errors as gptb_muon_step, and GPTB_ERR_INVALID_ARG for
 * count outside 1..64. */
size_t gptb_muon_batched_workspace_bytes(int count, int m, int n, int steps);
int gptb_muon_step_batched(int count, float* const* w, void* const* w_bf16, const float* const* g, float* const* buf,
                           float* const* v, int m, int n, const float* coeffs, int steps, float lr, float mu,
                           float beta2, float weight_decay, void* workspace, size_t workspace_bytes,
                           gptb_stream_t stream);

/* ---------------------------------------------------------- decode ----
 * One generation step of the inference engine (apidog.com/fr "Comment
 * Entraîner Votre Propre ChatGPT Pour 50€ ?", § 6 "Moteur d'inférence": a KV
 * cache filled at prefill, one new token per sequence per step): attention of
 * each sequence's newest token over its cache, with the training attention's
 * causal window and grouped-query heads (kv head of q head h = h / (H/H_kv)),
 * softmax scale 1/sqrt(128).
 *   q:       device bf16 [B, H, 128], the new tokens' (normalised, rotated) queries
 *   k_cache, v_cache: device bf16 [B, T_max, H_kv, 128] (row stride H_kv*128,
 *            sequence stride T_max*H_kv*128) holding positions 0..lens[b]-1 of
 *            sequence b, the new token's own k and v included
 *   lens:    device int32 [B]; a sequence with lens[b] outside 1..T_max gets
 *            o = 0 and lse = -inf
 *   window:  -1 = every cached key; W >= 0 keeps keys lens[b]-1-W .. lens[b]-1
 *   o:       device bf16 [B, H, 128]; lse: device fp32 [B, H] (natural log of
 *            the softmax denominator incl. its max) or NULL
 *   workspace: device, gptb_decode_workspace_bytes(B, H, T_max) bytes, 16-byte
 *            aligned (partial softmax sums of the key pieces; the keys of a
 *            sequence are split into pieces of 128, spread over the SMs and
 *            streamed through shared memory, then combined)
 * Errors: GPTB_ERR_INVALID_ARG (null / misaligned pointers, H % H_kv != 0),
 * GPTB_ERR_WORKSPACE (workspace too small), GPTB_ERR_UNSUPPORTED (more than
 * 8 query heads per kv head). */
size_t gptb_decode_workspace_bytes(int B, int H, int T_max);
int gptb_decode_attention(const void* q, const void* k_cache, const void* v_cache, const int32_t* lens, void* o,
                          float* lse, int B, int H, int Hkv, int T_max, int window, void* workspace,
                          size_t workspace_bytes, gptb_stream_t stream);

/* Element casts for data-parallel gradient buckets (bf16 on the wire):
 * y[i] = bf16(x[i] * scale) and y[i] = float(x[i]) * scale, n elements,
 * device pointers, round to nearest-even.  GPTB_ERR_INVALID_ARG for null
 * pointers or n < 0. */
int gptb_cast_f32_bf16(const float* x, void* y, long long n, float scale, gptb_stream_t stream);
int gptb_cast_bf16_f32(const void* x, float* y, long long n, float scale, gptb_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns GPTB_OK, GPTB_ERR_TIMEOUT if a bounded wait inside a kernel expired
 * (the kernel recorded it, drained and returned), GPTB_ERR_BAD_INPUT if a
 * kernel found invalid input data (a cross-entropy target outside
 * [0, vocab)), or GPTB_ERR_CUDA. */
int gptb_device_error(gptb_stream_t stream);

/* Self-test of the bounded waits: sets the wait limit to limit_ns, launches
 * one CTA that waits on an mbarrier nothing ever arrives on, synchronises,
 * restores the previous limit and returns the device status.  The expected
 * result is GPTB_ERR_TIMEOUT: the wait expired, the kernel recorded it and
 * returned, and the context stays usable.  No counterpart on the pages. */
int gptb_probe_bounded_wait(unsigned long long limit_ns, gptb_stream_t stream);

/* Wait limit (nanoseconds) of every bounded device wait; default 2 s.
 * Applies to kernels launched afterwards on the current device. */
int gptb_set_wait_limit_ns(unsigned long long ns);

/* Kernel accounting: every kernel this library launches increments a host
 * counter; with timing enabled, the GEMM launches are also bracketed by CUDA
 * events on their stream and their device time and FLOPs are accumulated. */
void gptb_reset_counters(void);
long long gptb_launch_count(void);
int gptb_set_gemm_timing(int enable);
/* GEMM device milliseconds and FLOPs since the last reset (syncs).  The
 * milliseconds are the time covered by the GEMM launches: the union of their
 * event intervals on one time base, i.e. the sum of their durations when no
 * two overlap and each instant counted once when launches on two streams run
 * together (the bf16 backward issues its weight-gradient GEMMs on a second
 * stream).  ms_fp8 / flops_fp8: the same for the GEMMs with e4m3 operands.
 * Any output pointer may be NULL. */
int gptb_gemm_timing(double* ms, double* flops, double* ms_fp8, double* flops_fp8, long long* launches);

/* Human-readable text for a return code. */
const char* gptb_error_string(int code);

#ifdef __cplusplus
}
#endif
#endif /* GPTBLOCK_H */

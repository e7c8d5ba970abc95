/*
 * nc.h -- C ABI of libnc.so: the nanochat GPT forward pass, from token ids to
 * per-token softcapped cross-entropy, on one B200 (sm_100a).
 *
 * The operation is the forward pass of "The Mathematics of Karpathy's
 * nanochat" (§High-Level Forward Pass and the sections it links), extended by
 * the smear gate and backout of the "nanochat depth sweep" model card
 * (Architecture list) and "Reading nanochat Source" (§5, Forward pass, shape
 * by shape).  The generation step of the same page (§Inference: Generating
 * Text, §Sampling Controls) runs on it: the logits of the last position only,
 * then a greedy or top-k / temperature draw.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers unless the argument says "host".
 *  - The library never allocates and never frees device memory: parameters
 *    are borrowed, scratch comes from a caller-provided workspace.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream) unless stated otherwise.
 *  - Arguments are validated on the host before any launch; a failed check
 *    returns a non-zero nc_status and launches nothing.  No call throws,
 *    exits or traps.
 *  - Data errors found on the device (token or target id out of range, a
 *    bounded wait that ran out) are clamped or skipped so that every access
 *    stays in bounds, and are recorded in a device status word that
 *    nc_get_status() returns.
 *  - Calls are thread-compatible: concurrent calls must not share a
 *    workspace.
 */
#ifndef NC_H_
#define NC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NC_MAX_LAYERS 64

typedef enum {
  NC_OK = 0,
  NC_ERR_ARG = 1,        /* null pointer or invalid scalar argument          */
  NC_ERR_SHAPE = 2,      /* unsupported or inconsistent sizes                */
  NC_ERR_ALIGN = 3,      /* pointer or stride not 16-byte aligned            */
  NC_ERR_CUDA = 4,       /* a CUDA runtime call failed (see nc_last_error)   */
  NC_ERR_DATA = 5,       /* device-side: token/target id out of range, or a
                            sampling uniform outside [0, 1)                   */
  NC_ERR_TIMEOUT = 6,    /* device-side: a bounded wait inside a kernel ran out */
  NC_ERR_WORKSPACE = 7   /* workspace missing or smaller than required       */
} nc_status;

typedef enum { NC_BF16 = 0, NC_FP32 = 1 } nc_dtype;

/* Model configuration.  Filled by nc_init_config(); every field may be
 * overridden by the caller before use. */
typedef struct nc_config {
  int n_layer;            /* L, the depth                                       */
  int n_embd;             /* C = ceil(64 L / 128) * 128 ([Math] §Architecture Overview) */
  int n_head;             /* H = C / 128                                        */
  int n_kv_head;          /* H_kv, a divisor of H: query head h reads k/v head h / (H / H_kv) */
  int head_dim;           /* D = 128 (the kernels require 128)                  */
  int vocab;              /* V = 32768                                          */
  int vocab_padded;       /* V rounded up to a multiple of 64 ([Source] §5.4)   */
  int mlp_hidden;         /* 4 C                                                */
  int max_T;              /* sequence length the windows are derived from      */
  int dtype;              /* nc_dtype: NC_BF16 (bf16 storage, fp32 accumulate) or NC_FP32 */
  int window[NC_MAX_LAYERS];  /* per-layer window w: key j visible to query i iff j <= i and i - j < w */
  int has_ve[NC_MAX_LAYERS];  /* value embedding on layer l iff l % 2 == (L - 1) % 2 */
  int backout_layer;      /* block whose output is subtracted before the head; -1 = none */
  int gate_channels;      /* 12: input channels of the VE and smear gates       */
  int smear;              /* 1 = smear gate on                                  */
  int gemm_impl;          /* 0 = tensor cores (tcgen05) in bf16 mode, 1 = CUDA-core GEMM */
  int attn_impl;          /* 0 = tensor cores (tcgen05) in bf16 mode, 1 = CUDA-core attention */
  int gemm_pair;          /* 1 = tcgen05 GEMMs on CTA pairs (cta_group::2, 256 x 256 tiles) where N % 256 == 0;
                            2 = the same, and for the MLP down-projection the k-blocks of its partial last
                            wave of tiles are split evenly over all CTA pairs (partial sums pass through the
                            workspace); measured slower than 1 at d24, kept as an option */
  float qk_alpha;         /* 1.15 ([Math] §QK-Norm with Sharpening)              */
  float softmax_scale;    /* 1/sqrt(D)                                          */
  float rope_base;        /* 100000                                             */
  float eps;              /* 1e-6, inside every RMSNorm's square root           */
  float softcap;          /* 15 ([Math] §Logit Softcap)                          */
  float ve_gate_scale;    /* 3 ([Math] §Value Embeddings)                        */
} nc_config;

/* Parameters of one block.  Matrices use the nn.Linear [out, in] row-major
 * layout (y = x W^T) in the config's dtype (bf16 or fp32). */
typedef struct nc_layer_params {
  const void* w_qkv;      /* [(H + 2 H_kv) D, C]: rows of W_Q, then W_K, then W_V */
  const void* w_o;        /* [C, H D]                                           */
  const void* w_fc1;      /* [4C, C]                                            */
  const void* w_fc2;      /* [C, 4C]                                            */
  const void* ve;         /* [V, H_kv D] value-embedding table, or NULL when has_ve == 0 */
  const float* ve_gate;   /* [H_kv, gate_channels] fp32, or NULL when has_ve == 0 */
} nc_layer_params;

typedef struct nc_params {
  nc_config cfg;
  const void* wte;            /* [V, C] token embedding                         */
  const void* lm_head;        /* [V_pad, C] untied head                         */
  const float* smear_gate;    /* [gate_channels] fp32                           */
  const float* resid_lambdas; /* [L] fp32, lambda_l                              */
  const float* x0_lambdas;    /* [L] fp32, mu_l                                  */
  float backout_lambda;       /* beta (host scalar)                             */
  nc_layer_params layer[NC_MAX_LAYERS];
  void* workspace;            /* device scratch of >= nc_workspace_bytes(cfg, max_tokens) */
  size_t workspace_bytes;
  int max_tokens;             /* B*T capacity the workspace was sized for       */
} nc_params;

/* Fill `cfg` (host out) for a model of depth `depth`, following [Math]
 * §Architecture Overview and §Sliding Window Pattern: the pattern string
 * ("SSSL", "L", ...) is tiled over the layers, 'L' -> window max_T, 'S' ->
 * short_window, and the last layer is always max_T.  backout_layer < 0 picks
 * L/2.  Pure host function.  Returns NC_ERR_ARG on a null pointer, a
 * non-positive size, a depth above NC_MAX_LAYERS or a pattern with characters
 * other than 'S'/'L'. */
int nc_init_config(nc_config* cfg, int depth, int max_T, int dtype, const char* window_pattern,
                   int short_window, int backout_layer);

/* Bytes of workspace nc_forward() needs for up to `max_tokens` = B*T tokens
 * (256-byte aligned sub-buffers).  Host function; 0 on invalid config. */
size_t nc_workspace_bytes(const nc_config* cfg, int max_tokens);

/* Zero `p` (host) and copy `cfg` into it.  The caller then sets the pointers. */
int nc_params_init(nc_params* p, const nc_config* cfg);

/* Forward pass ([Math] §High-Level Forward Pass, §Cross-Entropy Loss).
 *   tokens   [B, T] int32, ids in [0, V)
 *   targets  [B, T] int32, ids in [0, V) or -1 (= ignored)
 *   out_loss [B*T] fp32 per-token loss: logsumexp(zhat_t) - zhat_t[y_t], 0 where y_t == -1
 *   out_logits_opt [B*T, V] fp32 softcapped logits 15 tanh(z/15), or NULL
 *     (when NULL the logits are never written to memory in bf16 mode).
 * Requires B*T <= p->max_tokens, T <= cfg.max_T, C % 128 == 0, D == 128,
 * H % H_kv == 0, all pointers 16-byte aligned. */
int nc_forward(const nc_params* p, const int32_t* tokens, const int32_t* targets, int B, int T,
               float* out_loss, float* out_logits_opt, void* stream);

/* The same pass from HOST buffers: copies h_tokens/h_targets ([B, T] int32,
 * host) into the workspace, runs nc_forward() and copies the per-token loss
 * back into h_out_loss ([B*T] fp32, host).  Asynchronous on `stream` like every
 * call: h_out_loss holds the loss once the stream has been synchronised, and
 * the host buffers must stay valid until then.  With pinned host memory the
 * copies overlap other work on the GPU (consecutive calls on one stream
 * pipeline); with pageable memory the runtime may complete them before it
 * returns. */
int nc_forward_host(const nc_params* p, const int32_t* h_tokens, const int32_t* h_targets, int B,
                    int T, float* h_out_loss, void* stream);

/* Generation ([Math] §Inference: Generating Text, step 2): the forward pass
 * over tokens [B, T] (device int32, ids in [0, V)), then the head on the last
 * position of each row only:
 *   out_logits [B, V] fp32 (device), out_logits[b] = 15 tanh(z/15) with
 *   z = RMSNorm(x_L[b, T-1]) W_U^T (in bf16 mode the normalised row is
 *   rounded to bf16 before the product, as in nc_forward).
 * Same requirements as nc_forward, plus a width the head supports: in bf16
 * mode C a multiple of 64 up to 5168 (the tensor-core form) or C <= 2304,
 * in fp32 mode C <= 1280 (NC_ERR_SHAPE otherwise, before any launch); no
 * targets, no loss.
 * Status codes as nc_forward (NC_ERR_ARG for a NULL tokens/out_logits). */
int nc_last_logits(const nc_params* p, const int32_t* tokens, int B, int T, float* out_logits,
                   void* stream);

/* One token per row drawn from logits ([Math] §Sampling Controls):
 *   logits   [B, ldl] fp32 (device), first V entries of each row used
 *   uniforms [B] fp32 (device), u_b in [0, 1): the row's random number
 *   out_next [B] int32 (device)
 * temperature == 0: out_next[b] = argmax_v logits[b, v], the lowest index
 *   among equal maxima (greedy decoding).
 * temperature > 0: with top_k > 0 (and < V) the entries below the top_k-th
 *   largest value (ties counted) are dropped, so ties at that value are all
 *   kept; top_k == 0 or >= V keeps everything.  Weights
 *   w_v = exp((z_v - max z) / temperature); out_next[b] is the first v (in
 *   vocabulary order) whose cumulative weight exceeds u_b * sum_v w_v, i.e. a
 *   draw from P(v) = w_v / sum w by inversion of u_b.
 * fp32 throughout; a u_b outside [0, 1) sets NC_ERR_DATA in the status word
 * and is clamped.  NC_ERR_SHAPE: B <= 0, V <= 0, ldl < V, top_k < 0,
 * temperature < 0 or not finite.  No workspace; a row of V <= 40960 is staged
 * in shared memory, longer rows are read from global memory. */
int nc_sample(const float* logits, int B, int V, int ldl, float temperature, int top_k,
              const float* uniforms, int32_t* out_next, void* stream);

/* nc_last_logits() then nc_sample() on its logits (ldl = V): one generation
 * step.  out_logits [B, V] fp32 (device) is required and holds the logits
 * afterwards. */
int nc_generate_next(const nc_params* p, const int32_t* tokens, int B, int T, float temperature,
                     int top_k, const float* uniforms, int32_t* out_next, float* out_logits,
                     void* stream);

/* Bytes of the extra workspace nc_head_backward() needs for up to
 * max_tokens tokens: the per-token gradient of the logits in bf16
 * ([max_tokens, V_pad], 64 MiB per 1024 tokens at V = 32768) and one fp32
 * [max_tokens, C] buffer.  Host function; 0 on invalid config. */
size_t nc_head_backward_workspace_bytes(const nc_config* cfg, int max_tokens);

/* Backward pass of the head: the gradients of the mean cross-entropy
 * L = (1/|T|) sum_{t in T} (logsumexp(zhat_t) - zhat_t[y_t]), T = {t : y_t != -1},
 * with respect to the final residual stream and to the unembedding matrix
 * ("The Mathematics of Karpathy's nanochat", §Cross-Entropy Loss, §Logit
 * Softcap with d zhat/d z = 1 - tanh^2(z/15), §RMS Normalization; the chain
 * rule through these steps in reverse order):
 *   out_dx [B*T, C] fp32: dL/dx, x the final residual after backout (the
 *     input of the final RMSNorm);
 *   out_dw [V, C] fp32: dL/dW_U (rows V..V_pad-1 are not written).
 * It consumes what the forward pass left in p->workspace (bf16(x), the row
 * sums of squares of x, x itself and the per-row log-sum-exp), so it must
 * follow nc_forward(p, tokens, targets, B, T, ...) on the same stream with the
 * same p, B, T and targets, with no other call using that workspace in
 * between.  The logits are recomputed (one more head GEMM) and their gradient
 * is held in bf16 in bwd_workspace (>= nc_head_backward_workspace_bytes).
 * Then dL/dxn = dL/dz W_U and dL/dW_U = dL/dz^T xn run as tensor-core GEMMs
 * (xn in bf16 as the forward's head consumed it), and the RMSNorm backward
 * gives dL/dx.  With no valid target both gradients are 0.  bf16 mode with
 * tensor-core GEMMs only (NC_ERR_SHAPE otherwise); requirements and status
 * codes as nc_forward, NC_ERR_WORKSPACE for a missing or short bwd_workspace. */
int nc_head_backward(const nc_params* p, const int32_t* targets, int B, int T, float* out_dx, float* out_dw,
                     void* bwd_workspace, size_t bwd_workspace_bytes, void* stream);

/* Mean of loss[i] over i with targets[i] != -1 ([Math] §Cross-Entropy Loss),
 * written to *out_mean (device fp32); NaN when no target is valid.  n >= 0. */
int nc_loss_mean(const float* loss, const int32_t* targets, int n, float* out_mean, void* stream);

/* Workspace bytes nc_attention() needs (0 when rope_qknorm == 0). */
size_t nc_attention_workspace_bytes(int B, int T, int H, int Hkv, int D, int dtype, int rope_qknorm);

/* One attention layer ([Math] §QK-Norm with Sharpening, §Scaled Dot-Product
 * Attention with Sliding Window):
 *   q [B, T, H, D], k and v [B, T, H_kv, D] contiguous, in `dtype`;
 *   out [B, T, H, D] in `dtype`.
 *   With rope_qknorm = 1, q and k first get RoPE (base rope_base, position t
 *   within the row) and qhat = alpha * RMSNorm_D(RoPE(q)) (likewise k), written
 *   to the workspace; with 0 they are used as given.
 *   o_i = sum_j softmax_j(softmax_scale * qhat_i . khat_j) v_j over j <= i,
 *   i - j < window; window <= 0 or >= T means plain causal.
 * Query head h attends with k/v head h / (H / H_kv) (grouped-query attention).
 * Requires D == 128, H % H_kv == 0, softmax_scale > 0, eps >= 0, 16-byte aligned
 * pointers (NC_ERR_SHAPE / NC_ERR_ARG / NC_ERR_ALIGN otherwise). */
int nc_attention(const void* q, const void* k, const void* v, void* out, int B, int T, int H,
                 int Hkv, int D, int window, int rope_qknorm, float alpha, float softmax_scale,
                 float rope_base, float eps, int dtype, void* workspace, size_t workspace_bytes,
                 void* stream);

/* nc_attention without a workspace, for callers that have no way to obtain
 * device memory for scratch: code embedded in a host program whose memory is
 * managed by a runtime that does not expose an allocator, or a latency-bound
 * loop that must not call cudaMalloc (it can synchronise the device).  There is
 * no counterpart on the pages: this is a deployment convenience.
 *   Computes exactly what nc_attention(q, k, v, out, B, T, H, Hkv, D, window,
 *   rope_qknorm = 1, alpha, softmax_scale, rope_base, eps, dtype, ...) does,
 *   with the same argument meanings and requirements.
 *   Scratch: one array of nc_attention_noalloc_max_bytes() bytes (32 MiB) in
 *   device memory, defined in the library, held by every GPU that loads the
 *   library until the process exits.  Calls whose RoPE tables plus normalised
 *   q and k do not fit (about 2 * T * 256 + 2 * B * T * H * 128 * sizeof(dtype)
 *   bytes) return NC_ERR_WORKSPACE and launch nothing.  The call allocates and
 *   frees nothing itself.
 *   The first call on a device looks up the array's device address with that
 *   device current (host code cannot use the array's name as a device pointer);
 *   make that first call before any stream capture.
 *   All calls on a device share the array: every byte a call reads from it is
 *   written earlier by the same call, but calls that overlap on the GPU (other
 *   streams, or other threads) race on it and must be serialised by the caller. */
int nc_attention_noalloc(const void* q, const void* k, const void* v, void* out, int B, int T, int H,
                         int Hkv, int D, int window, float alpha, float softmax_scale, float rope_base,
                         float eps, int dtype, void* stream);

/* Size in bytes of nc_attention_noalloc's fixed scratch array. */
size_t nc_attention_noalloc_max_bytes(void);

/* Pass-2 attention of the looped ("routing") variant ("looped-nanochat-d24"
 * model card, What is the routing loop?): every pass-2 layer adds a causal
 * attention-logit prior from a pass-1 layer,
 *   logits_ij = softmax_scale * (q2_i . k2_j + g q1_i . k1_j),  g = softplus(gate_logit),
 * over the base model's visible keys (j <= i, i - j < window; window <= 0 or
 * >= T means plain causal), then o_i = sum_j softmax_j(logits_ij) v2_j.
 *   q2, q1 [B, T, H, D] and k2, k1, v2 [B, T, H_kv, D], bf16, contiguous: q and
 *     k are the features as they enter the attention (after RoPE and QK-norm
 *     of their pass); query head h reads k/v head h / (H / H_kv);
 *   out [B, T, H, D] bf16.
 * As on the card, the prior never forms a T x T matrix: it is one QK^T over
 * the augmented width [q2 | g q1] . [k2 | k1] on the tensor cores.  g q1 is
 * written (bf16) to `workspace` (>= nc_routing_attention_workspace_bytes).
 * bf16 only; D == 128, H % H_kv == 0, softmax_scale > 0, finite gate_logit,
 * 16-byte aligned pointers (NC_ERR_SHAPE / NC_ERR_ARG / NC_ERR_ALIGN /
 * NC_ERR_WORKSPACE otherwise). */
size_t nc_routing_attention_workspace_bytes(int B, int T, int H, int D);
int nc_routing_attention(const void* q2, const void* k2, const void* v2, const void* q1, const void* k1, void* out,
                         int B, int T, int H, int Hkv, int D, int window, float gate_logit, float softmax_scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/* StairFormer nesting pieces ("Fully Nested Transformers" README: block
 * lower triangular weights keep the residual stream of smaller models a
 * prefix of larger models', and PrefixRMSNorm keeps normalisation from
 * leaking information backward down the hierarchy).  A width C is cut into k
 * nested blocks, `widths` (host array of k ints, 1 <= k <= 8, each a positive
 * multiple of 64, summing to C); C_a = widths[0] + ... + widths[a].  The
 * j-front submodel is the first j blocks.  NC_ERR_SHAPE on other widths.
 *
 * nc_prefix_rmsnorm: block a of the output is block a of x divided by the RMS
 * of x's prefix up to C_a:
 *   out[m, c] = x[m, c] / sqrt(mean(x[m, :C_a]^2) + eps),  C_{a-1} <= c < C_a.
 * x [M, C] fp32, out [M, C] bf16 (out_bf16 != 0) or fp32, row-major, 16-byte
 * aligned device pointers (NC_ERR_ALIGN).  With one block it is RMSNorm. */
int nc_prefix_rmsnorm(const float* x, int M, int C, const int* widths, int k, float eps, void* out, int out_bf16,
                      void* stream);

/* nc_btl_linear: y = x W^T with W [C_out, C_in] block lower triangular:
 * output block a (columns below C_out_a) reads input blocks b <= a only
 * (elements below C_in_a).  W is stored dense, row-major, and its dead blocks
 * must hold zeros: each 256-column output tile contracts over the input prefix
 * its last column reads, so dead blocks beyond it are never loaded, and those
 * inside it are multiplied as the zeros they are.  x [M, C_in] bf16, W bf16,
 * y [M, C_out] fp32; in_widths and out_widths: k block widths each.  C_out must
 * be a multiple of 256 (NC_ERR_SHAPE); 16-byte aligned pointers. */
int nc_btl_linear(const void* x, const void* w, float* y, int M, int C_in, int C_out, const int* in_widths,
                  const int* out_widths, int k, void* stream);

/* nc_prefix_ce: per-token softcapped cross-entropy of every j-front
 * submodel, j = 1..k: its logits use the first C_j columns of the head on the
 * normalised prefix,
 *   z_j = PrefixRMSNorm(x)[:, :C_j] W_U[:, :C_j]^T,  zhat_j = cap tanh(z_j / cap),
 *   out_loss[(j - 1) M + m] = logsumexp_v zhat_j[m, v] - zhat_j[m, y_m]
 * over v < V (0 where y_m = -1; out-of-range targets are flagged as in
 * nc_forward).  x [M, C] fp32; w_u [V_pad, C] bf16 (rows V.. V_pad - 1 are
 * read but excluded from the sums); targets [M] int32; out_loss [k, M] fp32.
 * PrefixRMSNorm(x) is held in bf16 (the head GEMM's operand) in `workspace`
 * (>= nc_prefix_ce_workspace_bytes).  V_pad a multiple of 256 (NC_ERR_SHAPE);
 * 16-byte aligned pointers. */
size_t nc_prefix_ce_workspace_bytes(int M, int C, int V_pad);
int nc_prefix_ce(const float* x, const void* w_u, const int32_t* targets, float* out_loss, int M, int C, int V,
                 int V_pad, const int* widths, int k, float eps, float cap, void* workspace, size_t workspace_bytes,
                 void* stream);

/* Synchronise `stream`, read the device status word (an OR of
 * 1 << NC_ERR_DATA and 1 << NC_ERR_TIMEOUT bits set by kernels since the last
 * read), clear it, and return NC_OK, NC_ERR_DATA or NC_ERR_TIMEOUT (timeout
 * wins).  *out_bits (host, may be NULL) receives the raw bits. */
int nc_get_status(void* stream, int* out_bits);

/* Static description of a status code. */
const char* nc_status_string(int status);

/* Text of the last CUDA error seen by this thread (empty if none). */
const char* nc_last_error(void);

/* Number of kernel launches issued by the last nc_forward() / nc_attention()
 * on this thread. */
int nc_last_launch_count(void);

/* Test hook for the device-side timeout path (process-wide; not for normal
 * use).  With gemm_pair == 2 the MLP down-projection's partial last wave of
 * tiles is split over CTA pairs, and the pair that finishes a tile waits for
 * its contributors' flags (a generation number per launch).  With skew != 0
 * that wait expects generation + skew, which never arrives: after
 * wait_limit_ms the kernel records NC_ERR_TIMEOUT in the status word, skips
 * the wait and completes (its output is then not the model's).  wait_limit_ms
 * bounds that wait in every case (default 1000; nc_set_flag_wait_test(0,
 * 1000) restores normal operation).  Waits on in-flight copies and MMAs keep
 * their own one-second limit.  NC_ERR_ARG for skew < 0 or a limit outside
 * (0, 1000] ms.  There is no counterpart on the pages. */
int nc_set_flag_wait_test(int skew, double wait_limit_ms);

/* Optional per-launch device timing for profiling.  `events` is an array of
 * 2 * capacity cudaEvent_t created by the caller (passed as void*), `kinds`
 * an int array of `capacity`.  While set, every launch by this thread whose
 * kernel kind k has bit k set in kind_mask records events[2i] before and
 * events[2i+1] after it on the call's stream, and kinds[i] = k, for i = 0, 1,
 * ... up to capacity.  Calling again (or with events == NULL, which disables
 * it) restarts the count.  Kinds: 0 embed_norm_smear, 1 rmsnorm, 2 rope_table,
 * 3 rope_qknorm, 4 gemm_tcgen05, 5 gemm_cuda_core, 6 attention_tcgen05,
 * 7 attention_cuda_core, 8 ce_combine, 9 ce_rows, 10 loss_mean, 11 last_logits,
 * 12 sample, 13 gemm_tcgen05_bwd, 14 head_bwd_rows, 15 prefix_rmsnorm.
 * Returns NC_ERR_ARG if events != NULL with kinds == NULL or capacity <= 0. */
int nc_set_launch_timing(void** events, int* kinds, int capacity, unsigned kind_mask);

/* Event pairs recorded since the last nc_set_launch_timing() on this thread. */
int nc_launch_timing_count(void);

/* Name of a kernel kind ("unknown" out of range). */
const char* nc_kernel_name(int kind);

/* sizeof of the ABI structs, for bindings to check their mirrors:
 * which = 0 -> nc_config, 1 -> nc_layer_params, 2 -> nc_params; 0 otherwise. */
size_t nc_sizeof(int which);

#ifdef __cplusplus
}
#endif

#endif /* NC_H_ */

/*
 * dg.h - C ABI of the B200 canvas-denoising library (libdg.so).
 *
 * The library runs the block-autoregressive discrete-diffusion denoising step
 * of a DiffusionGemma-style model on one NVIDIA B200 (sm_100a):
 *   - a 256-token canvas attends bidirectionally to itself and to the causal
 *     KV cache of the committed prefix,
 *   - is projected to vocabulary logits,
 *   - is resampled (Philox-keyed Gumbel-max under a linear 0.8 -> 0.4
 *     temperature schedule, top-k commit, threshold re-noise, adaptive stop),
 *   - and, once stopped, has its K/V appended to the cache.
 * Sources: "DiffusionGemma Guia do Desenvolvedor para Decodificacao Paralela a
 * 1000+ Tokens/s", sections "Difusao de Estado Uniforme" and "Block
 * Autoregressive Diffusion para Sequencias Longas"; aiexpert.news "Google's
 * DiffusionGemma Atinge 1.000 Tokens por Segundo", architecture paragraph;
 * Google docs page "DiffusionGemma", bullet "Arquitetura de
 * codificador-decodificador" and table "Configuracao de exibicao recomendada".
 *
 * Conventions (all entry points):
 *   - Every function returns an int status (enum dg_status).  DG_OK is 0.
 *     dg_status_string() names a status; dg_last_error() gives a
 *     thread-local detail message for the last failure in this thread.
 *   - No C++ exception crosses this boundary.
 *   - Ownership: the caller allocates and owns every device buffer.  The
 *     library never allocates device memory (the driver-side resources of
 *     the CUDA graph that dg_denoise_block instantiates aside; see there).
 *     Scratch space comes from a caller-supplied workspace whose size the
 *     *_workspace_bytes() queries return.  Host arrays passed in (pointer
 *     tables, structs) are read during the call only.
 *   - One host thread at a time: the library keeps a little process-wide
 *     state (kernel attributes set once per device, a capture stream per
 *     device).  Calls may target any device: the current CUDA device is the
 *     one whose memory the pointers refer to.
 *   - All device work is enqueued on the caller's stream (a cudaStream_t passed
 *     as void*; NULL is the legacy default stream) and is asynchronous, except
 *     where a function says it synchronises.  Results are deterministic: the
 *     same inputs and seed give the same bits.
 *   - Argument errors (null pointers, unsupported shapes, misalignment, a too
 *     small workspace) are detected on the host before any launch and return
 *     an error with nothing enqueued.
 *   - Errors found on the device (a bounded wait that expired, a device-side
 *     bounds check) set a per-device error word instead of faulting.
 *     dg_check_device_errors() synchronises the stream, reads and clears it.
 *   - Device pointers must be 16-byte aligned; matrices are row-major with the
 *     last dimension contiguous.  bf16 means IEEE bfloat16.
 *   - Two environment variables change how work is scheduled, never what it
 *     computes: DG_PDL=0 launches kernels without programmatic dependent
 *     launch (each starts once its predecessor has finished), DG_GRAPHS=0
 *     makes dg_denoise_block launch every step directly instead of replaying
 *     a CUDA graph.  Both are read once per process.
 */
#ifndef DG_H_
#define DG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum dg_status {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,
  DG_ERR_UNSUPPORTED_SHAPE = 2,
  DG_ERR_ALIGNMENT = 3,
  DG_ERR_WORKSPACE_TOO_SMALL = 4,
  DG_ERR_CUDA = 5,
  DG_ERR_TIMEOUT = 6,
  DG_ERR_DEVICE_CHECK = 7
};

/* Attention key masks over [cached prefix ; new rows]. */
enum dg_mask_mode {
  DG_MASK_BIDIR = 0,  /* denoising canvas: every prefix key and every new row */
  DG_MASK_CAUSAL = 1  /* prefill / block re-encode: every prefix key, new rows j <= i */
};

/* What happens to uncommitted positions that are not selected in a step. */
enum dg_unselected_policy {
  DG_UNSELECTED_KEEP = 0,    /* take the step's sample, stay uncommitted (default) */
  DG_UNSELECTED_RENOISE = 1  /* take a fresh uniform token, stay uncommitted */
};

/* Epilogues of dg_linear. */
enum dg_epilogue {
  DG_EPI_F32 = 0,        /* out fp32 [M,N] = x w^T */
  DG_EPI_BF16 = 1,       /* out bf16 [M,N] = x w^T */
  DG_EPI_GELU_BF16 = 2,  /* out bf16 [M,N] = gelu_erf(x w^T) */
  DG_EPI_RESID_F32 = 3   /* out fp32 [M,N] += x w^T (residual add in place) */
};

typedef struct dg_model_cfg {
  int d;           /* model width */
  int n_layers;
  int n_q_heads;   /* Hq */
  int n_kv_heads;  /* Hkv; Hq % Hkv == 0; query head h reads kv head h / (Hq/Hkv) */
  int head_dim;    /* hd in {64, 128} */
  int ffn;         /* MLP width F */
  int vocab;       /* V, a multiple of 128 */
  float eps;       /* RMSNorm epsilon (the gain is 1) */
} dg_model_cfg;

/* One layer's bf16 weights, [out_features, in_features] row-major. */
typedef struct dg_layer_weights {
  const void* w_qkv;   /* [(Hq + 2 Hkv) hd, d], rows [Q heads | K heads | V heads] */
  const void* w_o;     /* [d, Hq hd] */
  const void* w_up;    /* [F, d] */
  const void* w_down;  /* [d, F] */
} dg_layer_weights;

/* e4m3 copies of a layer's projection weights (dg_quantize_e4m3 per tensor). */
typedef struct dg_layer_weights_e4m3 {
  const uint8_t* w_qkv;
  const uint8_t* w_o;
  const uint8_t* w_up;
  const uint8_t* w_down;
  const float* scales;  /* device [4]: the scales of w_qkv, w_o, w_up, w_down */
} dg_layer_weights_e4m3;

typedef struct dg_model {
  dg_model_cfg cfg;
  const void* embed;                /* bf16 [V, d] */
  const void* unembed;              /* bf16 [V, d] (untied) */
  const dg_layer_weights* layers;   /* host array of cfg.n_layers entries */
  /* Optional e4m3 copy of the unembedding (dg_quantize_e4m3, one tensor
   * scale): when set (V % 256 == 0, d % 128 == 0), the denoising loop's
   * unembedding + sampler step runs on FP8 operands, the hidden states
   * quantised per token each step.  NULL: bf16. */
  const uint8_t* unembed_e4m3;      /* e4m3 [V, d] */
  const float* unembed_scale;       /* device scalar */
  /* Optional e4m3 projections: when set, every projection of every forward
   * pass (prefill, denoising, block re-encode) runs on FP8 operands, its bf16
   * input quantised per token just before it.  Host array of cfg.n_layers
   * entries, or NULL (bf16). */
  const dg_layer_weights_e4m3* layers_e4m3;
} dg_model;

/* Which uncommitted positions a step commits.
 * DG_SELECT_TOP_K: the commit_k of largest log confidence (aiexpert.news
 *   architecture paragraph: 15-20 confident tokens locked per pass).
 * DG_SELECT_ENTROPY: Google docs table "Configuracao de exibicao recomendada",
 *   row "Selecao de token" (entropy limit 0.1): the uncommitted positions in
 *   increasing entropy (ties to the lower position), as long as their summed
 *   entropy stays <= entropy_bound, and at least the first one. */
enum dg_selection { DG_SELECT_TOP_K = 0, DG_SELECT_ENTROPY = 1 };

/* Sampler settings.  dg_sampler_defaults() fills the published values. */
typedef struct dg_sampler_cfg {
  int max_steps;        /* step cap per canvas (48) */
  float t_start;        /* temperature at step 0 (0.8) */
  float t_end;          /* temperature at step max_steps-1 (0.4) */
  int commit_k;         /* positions committed per step (16) */
  float renoise_conf;   /* re-noise committed tokens whose softmax confidence is below (0.05) */
  float stop_entropy;   /* adaptive stop: mean canvas entropy below, in nats (0.005) */
  int unselected_policy;/* enum dg_unselected_policy */
  int selection;        /* enum dg_selection (DG_SELECT_TOP_K) */
  float entropy_bound;  /* DG_SELECT_ENTROPY: summed-entropy limit, nats (0.1) */
} dg_sampler_cfg;

/* Per-step sampler diagnostics: caller-owned device arrays; any may be NULL.
 * near_ties counts, per sequence, the step's decisions that lie within 1e-4
 * (nats) of flipping, so that a caller comparing two implementations can
 * tell a rounding-level disagreement from a real one:
 *   [b*3 + 0] positions at the commit cut: with top-k, when the k-th and
 *             (k+1)-th largest log confidences of the uncommitted positions
 *             differ by less than 1e-4, the uncommitted positions within 1e-4
 *             of their midpoint; with DG_SELECT_ENTROPY, the last selected and
 *             first unselected positions when a sum of entropies through
 *             either lies within 1e-4 of entropy_bound or their entropies
 *             differ by less than 1e-4 (the last selected alone when every
 *             uncommitted position was selected with a sum within 1e-4 of it);
 *   [b*3 + 1] committed positions whose log confidence is within 1e-4 of
 *             ln(renoise_conf);
 *   [b*3 + 2] 1 when the mean entropy is within 1e-4 of stop_entropy.
 * The top-2 margins of the raw logits and of the Gumbel-perturbed scores are
 * not counted: the row pass keeps only each position's leader. */
typedef struct dg_step_out {
  int32_t* x_hat;     /* [B, C] the Gumbel-max sample of each position */
  int32_t* argmax;    /* [B, C] argmax of the raw logits (the step's "prediction") */
  float* logconf;     /* [B, C] log softmax confidence (tempered) of the token at stake */
  float* entropy;     /* [B, C] tempered entropy, nats */
  uint8_t* flags;     /* [B, C] bit0: committed this step, bit1: re-noised this step */
  int32_t* near_ties; /* [B, 3] near-tie counters (above); untouched for stopped sequences */
} dg_step_out;

/*
 * Generation state of a batch of B sequences.  All pointers are device
 * pointers owned by the caller, except the two host pointer tables.
 */
typedef struct dg_state {
  int batch;              /* B */
  int lmax;               /* cache capacity in rows */
  int canvas;             /* C, the canvas length (256) */
  int cache_len_host;     /* host mirror of the cache length, equal for every sequence */
  void* const* k_cache;   /* host table [n_layers] of bf16 [B, Hkv, lmax, hd] */
  void* const* v_cache;   /* host table [n_layers] of bf16 [B, Hkv, lmax, hd] */
  int32_t* cache_len;     /* [B] rows of the cache in use */
  int32_t* tok;           /* [B, C] canvas tokens */
  uint8_t* committed;     /* [B, C] 1 = committed */
  int32_t* prev_argmax;   /* [B, C] previous step's prediction (-1: none) */
  int32_t* seq_status;    /* [B] 0 = running; s + 1 once stopped after step s */
  int32_t* step;          /* [1] current step index of the canvas */
} dg_state;

const char* dg_status_string(int status);
const char* dg_last_error(void);
int dg_version(void);
/* Number of kernels this library has enqueued since it was loaded (all devices). */
unsigned long long dg_launch_count(void);
void dg_sampler_defaults(dg_sampler_cfg* cfg);

/* Synchronise `stream`, read and clear the device error word.
 * Returns DG_OK, DG_ERR_TIMEOUT (a bounded wait expired) or DG_ERR_DEVICE_CHECK
 * (a device-side bounds check failed); *code_out (may be NULL) gets the raw word. */
int dg_check_device_errors(void* stream, uint32_t* code_out);

/*
 * dg_canvas_attn - grouped-query attention of Lq new rows over
 * [cached prefix ; new rows] (the canvas attention of the denoising step, and
 * the causal attention of prefill and block re-encode).
 * Source: aiexpert.news architecture paragraph (bidirectional attention on the
 * canvas, causal prefill into the KV cache); Guia do Desenvolvedor, bullet
 * "Propagacao de Contexto Bidirecional".
 *   out[b,i,h,:] = softmax_j(q[b,i,h,:] . key_j * scale) value_j over keys
 *   j in { prefix rows 0..cache_len[b]-1 of kv head g } U { new rows allowed
 *   by mask_mode }, g = h / (Hq/Hkv).  No positional encoding.
 * Layouts (bf16):
 *   q      [B, Lq, ldq]    head h at columns h*hd .. h*hd+hd-1
 *   k_new, v_new [B, Lq, ldkv]  kv head g at columns g*hd
 *   k_cache, v_cache [B, Hkv, lmax, hd]
 *   out    [B, Lq, ldo]    head h at columns h*hd
 *   lse    fp32 [B, Hq, Lq] natural-log sum of exp of the scaled scores (may be NULL)
 *   cache_len: device [B]; every value must be <= max_prefix (host bound used
 *   to plan the split over keys).
 * Cached rows from cache_len[b] up to the next multiple of 128 are read and
 * weighted by zero: they must hold finite values (a zeroed cache does).
 * Requires hd in {64,128}, Hq % Hkv == 0, Lq >= 1, lmax >= max_prefix,
 * ldq/ldkv/ldo multiples of 8.  Workspace: dg_canvas_attn_workspace_bytes().
 */
int dg_canvas_attn(const void* q, int ldq, const void* k_new, const void* v_new, int ldkv,
                   const void* k_cache, const void* v_cache, const int32_t* cache_len,
                   int max_prefix, int lmax, void* out, int ldo, float* lse,
                   int B, int Hq, int Hkv, int Lq, int hd, float scale, int mask_mode,
                   void* workspace, size_t workspace_bytes, void* stream);
size_t dg_canvas_attn_workspace_bytes(int B, int Hq, int Hkv, int Lq, int hd, int max_prefix);

/*
 * dg_canvas_attn_e4m3 - dg_canvas_attn on e4m3 operands (the FP8 attention of
 * FP8 serving; aiexpert.news, "Google's DiffusionGemma Atinge 1.000 Tokens por
 * Segundo", throughput paragraph, quotes FP8 on one H200 without a recipe).
 * This library's recipe, with the codes of dg_quantize_e4m3:
 *   s[i, j] = scale * q_scale[b*Lq+i] * k_scale * sum_d dec(q)[d] dec(key_j)[d]
 *   p[i, j] = exp(s[i, j] - m_i), m_i a running maximum of row i that lags the
 *             row's by at most a factor 2^8 (p <= 256)
 *   out[b,i,h,:] = v_scale * sum_j e4m3(p[i, j]) dec(value_j) / sum_j p[i, j]
 * i.e. both products are 8-bit MMAs with fp32 accumulation, the probabilities
 * enter the value product as e4m3 values and the normaliser unrounded.  Keys,
 * mask, GQA mapping, split plan and lse are those of dg_canvas_attn.
 * Layouts (one byte per e4m3 code):
 *   q        [B, Lq, ldq]        head h at columns h*128; q_scale device fp32
 *                                [B*Lq], one per token (dg_quantize_e4m3 per row)
 *   k_new    [B, Lq, ldkv]       kv head g at columns g*128
 *   vt_new   [B, Hkv, 128, ldvt] V of the new rows transposed: row (b, g, d)
 *                                holds d of keys 0..Lq-1
 *   k_cache  [B, Hkv, lmax, 128]
 *   vt_cache [B, Hkv, 128, lmax] the cached V transposed the same way
 *   k_scale, v_scale: device fp32 scalars, one for prefix and new rows together
 *   out      bf16 [B, Lq, ldo]; lse fp32 [B, Hq, Lq] or NULL
 * Every scale must be positive and finite.  Cached keys from cache_len[b] up to
 * the next multiple of 128 are read and weighted by zero: they must hold finite
 * codes (a zeroed cache does).  Requires hd == 128, ldq, ldkv, ldvt and lmax
 * multiples of 16, ldvt >= Lq, ldo a multiple of 8.  Workspace:
 * dg_canvas_attn_workspace_bytes(B, Hq, Hkv, Lq, 128, max_prefix).
 */
int dg_canvas_attn_e4m3(const uint8_t* q, int ldq, const float* q_scale, const uint8_t* k_new,
                        int ldkv, const uint8_t* vt_new, int ldvt, const uint8_t* k_cache,
                        const uint8_t* vt_cache, const float* k_scale, const float* v_scale,
                        const int32_t* cache_len, int max_prefix, int lmax, void* out, int ldo,
                        float* lse, int B, int Hq, int Hkv, int Lq, int hd, float scale,
                        int mask_mode, void* workspace, size_t workspace_bytes, void* stream);

/*
 * dg_unembed - vocabulary logits of the normalised final hidden states (the
 * "diffusion head" of aiexpert.news architecture paragraph; untied).
 *   logits[m, v] = sum_k h[m, k] w_u[v, k]
 * h bf16 [M, d]; w_u bf16 [V, d]; logits fp32 [M, V].  V % 128 == 0,
 * d % 64 == 0.  Needs no workspace (pass NULL, 0).
 */
int dg_unembed(const void* h, const void* w_u, float* logits, int M, int d, int V,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * dg_linear - the layer projections of the stack (QKV, output, MLP up/down;
 * aiexpert.news architecture paragraph, with the dense GELU MLP standing in
 * for the expert FFN):
 *   y[m, n] = sum_k x[m, k] w[n, k], then the epilogue (enum dg_epilogue).
 * x bf16 [M, K]; w bf16 [N, K]; out per epilogue.  N % 128 == 0, K % 64 == 0.
 * Few tokens run on a GEMM whose K is split over a thread-block cluster; many
 * tokens (N % 256 == 0 and at least 74 output tiles of 256 x 256, or 48 with
 * M >= 1536; K at least four 128-byte k-blocks) on a persistent grid of CTA
 * pairs.  The path depends on the shape only, so a
 * shape always gives the same bits; the two paths sum K in different orders.
 * Needs no workspace: dg_linear_workspace_bytes() returns 0 (the split-K
 * partial sums stay in the cluster's shared memory); pass NULL, 0.
 */
int dg_linear(const void* x, const void* w, void* out, int M, int N, int K, int epilogue,
              void* workspace, size_t workspace_bytes, void* stream);
size_t dg_linear_workspace_bytes(int M, int N, int K);

/* Execution plans of the projections (host-side queries; no device work). */
enum dg_linear_plan {
  DG_PLAN_SPLIT_K = 0,  /* tcgen05 GEMM, K split over a thread-block cluster */
  DG_PLAN_PAIRS = 1     /* persistent grid of CTA pairs, 256 x 256 tiles */
};

/*
 * dg_linear_plan_of - the plan dg_linear (e4m3 = 0) or dg_linear_e4m3
 * (e4m3 != 0) uses for this shape; -1 for a shape they reject.
 * dg_model_residual_on_pairs - 1 when a forward pass of the model over M
 * tokens runs both residual projections (output, K = Hq hd; MLP down, K = F)
 * on CTA pairs, 0 otherwise; -1 for a null cfg or M < 1.  Each projection
 * takes the plan of its own shape.
 */
int dg_linear_plan_of(int M, int N, int K, int e4m3);
int dg_model_residual_on_pairs(const dg_model_cfg* cfg, int M, int e4m3);

/*
 * dg_sample_commit - one sampler step over logits [B, C, V] fp32.
 * Source: Google docs table "Configuracao de exibicao recomendada" (step cap,
 * linear temperature schedule, adaptive stop on entropy + two identical
 * predictions); aiexpert.news architecture paragraph (confident tokens locked
 * per pass, low-confidence positions re-noised); Guia do Desenvolvedor bullet
 * "Correcao de Erros via Re-Noising".
 * Per position, with T = t_start + (t_end - t_start) * step / (max_steps - 1)
 * and z = logits / T: entropy of softmax(z); argmax of the raw logits; the
 * Gumbel-max sample x_hat = argmax(z + g), g = -ln(-ln u), u from
 * Philox4x32-10 keyed (seed, b) with counter (v >> 2, pos | 0 << 24, step,
 * block), word v & 3, u = (2 (r >> 9) + 1) 2^-24; log confidence
 * lambda = z[x] - logsumexp(z) (x = x_hat if uncommitted, else the current token).
 * Then: commit the min(k, #uncommitted) uncommitted positions of largest
 * lambda (ties to the lower position) to x_hat (or, with selection =
 * DG_SELECT_ENTROPY, the entropy-bounded prefix described at enum dg_selection); re-noise committed positions
 * with lambda < ln(renoise_conf) to a uniform token (Philox tag 1, counter
 * (0, pos | 1 << 24, step, block), token = (r * V) >> 32) and uncommit them;
 * unselected uncommitted positions follow unselected_policy.  Stop when every
 * position is committed, or when mean entropy < stop_entropy and the argmax
 * equals the previous step's everywhere (step >= 1), or at step max_steps - 1;
 * the latter two commit every remaining position to x_hat and skip re-noise.
 * In/out (device): tok, committed, prev_argmax [B, C]; seq_status [B]
 * (sequences with a nonzero status are left untouched).  out may be NULL.
 * C <= 1024, V % 4 == 0.  Workspace: dg_sample_commit_workspace_bytes().
 */
int dg_sample_commit(const float* logits, int32_t* tok, uint8_t* committed,
                     int32_t* prev_argmax, int32_t* seq_status, const dg_sampler_cfg* cfg,
                     uint32_t seed, int block, int step, int B, int C, int V,
                     const dg_step_out* out, void* workspace, size_t workspace_bytes,
                     void* stream);
size_t dg_sample_commit_workspace_bytes(int B, int C, int V);

/*
 * dg_unembed_sample_commit - dg_unembed followed by dg_sample_commit, fused:
 * the logits h w_u^T are formed tile by tile on the tensor cores and reduced
 * to the sampler's per-position statistics in registers, so they never reach
 * memory.  Same sources, definitions and in/out state as dg_sample_commit,
 * with logits[b, i, v] = sum_k h[b*C + i, k] w_u[v, k].
 * h bf16 [B*C, d] (already normalised); w_u bf16 [V, d].  V % 256 == 0,
 * d % 64 == 0, C <= 1024.  Workspace: dg_unembed_sample_commit_workspace_bytes().
 * The statistics are merged in a different order than dg_sample_commit's,
 * so sums agree to rounding and decisions agree except at near-ties.
 */
int dg_unembed_sample_commit(const void* h, const void* w_u, int d, int32_t* tok,
                             uint8_t* committed, int32_t* prev_argmax, int32_t* seq_status,
                             const dg_sampler_cfg* cfg, uint32_t seed, int block, int step,
                             int B, int C, int V, const dg_step_out* out, void* workspace,
                             size_t workspace_bytes, void* stream);
size_t dg_unembed_sample_commit_workspace_bytes(int B, int C, int V);

/*
 * FP8 (e4m3) unembedding.  The pages quote FP8 checkpoints without fixing a
 * recipe; this library's: e4m3 (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, largest finite value 448), nearest value with ties to
 * even, saturating; scale = max |x| / 448 in fp32 (1 for an all-zero block).
 *
 * dg_quantize_e4m3 - in bf16 [rows, cols] -> out e4m3 [rows, cols] and
 *   scales: per_row != 0: one per row (scales[rows]); per_row == 0: one for
 *   the tensor (scales[0]).  x ~= scale * e4m3_value.  cols % 8 == 0.
 * dg_unembed_e4m3 - logits[m, v] = hs[m] * ws * sum_k dec(h_q[m, k]) dec(w_q[v, k])
 *   (fp32 accumulate of exact products); h_scale device [M], w_scale device
 *   scalar.  V % 256 == 0, d % 128 == 0.
 * dg_unembed_sample_commit_e4m3 - dg_unembed_sample_commit with the logits of
 *   dg_unembed_e4m3.  Workspace: dg_unembed_sample_commit_workspace_bytes().
 * dg_linear_e4m3 - dg_linear on e4m3 operands: x_q [M, K] codes with per-row
 *   scales x_scale (device [M]), w_q [N, K] codes with one scale w_scale
 *   (device scalar); acc[m, n] = x_scale[m] w_scale sum_k dec(x_q[m, k])
 *   dec(w_q[n, k]) (fp32 accumulation of exact products), then the epilogue
 *   of dg_linear, on the same two paths (kind::f8f6f4 MMAs).  N % 128 == 0,
 *   K % 128 == 0.  No workspace.
 */
int dg_quantize_e4m3(const void* in, int rows, int cols, int per_row, uint8_t* out,
                     float* scales, void* stream);
int dg_linear_e4m3(const uint8_t* x_q, const float* x_scale, const uint8_t* w_q,
                   const float* w_scale, void* out, int M, int N, int K, int epilogue,
                   void* stream);
int dg_unembed_e4m3(const uint8_t* h_q, const float* h_scale, const uint8_t* w_q,
                    const float* w_scale, float* logits, int M, int d, int V, void* stream);
int dg_unembed_sample_commit_e4m3(const uint8_t* h_q, const float* h_scale, const uint8_t* w_q,
                                  const float* w_scale, int d, int32_t* tok, uint8_t* committed,
                                  int32_t* prev_argmax, int32_t* seq_status,
                                  const dg_sampler_cfg* cfg, uint32_t seed, int block, int step,
                                  int B, int C, int V, const dg_step_out* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * dg_sample_commit_noalloc - dg_sample_commit without a workspace argument.
 * No page describes it: this is a library convenience.  It serves
 * callers that cannot allocate device memory - a plugin whose host owns every
 * device allocation, or code enqueueing work during stream capture, where
 * cudaMalloc is not permitted.  Its scratch lives in a fixed 4 MiB static
 * device array that every GPU loading the library keeps until process exit;
 * nothing is allocated per call (no cudaMalloc, cudaFree or allocating library
 * routine).  Sizes whose scratch exceeds 4 MiB (dg_sample_commit_workspace_bytes
 * of B, C, V: 32 bytes per position and vocabulary chunk, the chunks 131072
 * entries once there are 16 or more per SM, so at C = 256, V = 262144 up to
 * B = 256) return DG_ERR_UNSUPPORTED_SHAPE.  The
 * first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for the life
 * of the process; make that first call before any stream capture.  A device
 * reset (cudaDeviceReset) between calls is not supported: the module may be
 * reloaded elsewhere and the kept address would be stale.  All calls share the one array and it
 * keeps the last call's contents (every slot read is written earlier in the
 * same call, so nothing needs clearing); calls that overlap on the GPU - on
 * different streams, or from different threads - race on it and must be
 * serialised by the caller.  Arguments and results as dg_sample_commit.
 */
int dg_sample_commit_noalloc(const float* logits, int32_t* tok, uint8_t* committed,
                             int32_t* prev_argmax, int32_t* seq_status, const dg_sampler_cfg* cfg,
                             uint32_t seed, int block, int step, int B, int C, int V,
                             const dg_step_out* out, void* stream);

/*
 * dg_kv_block_commit - append a finished block's per-layer K/V to the cache
 * ("Guia do Desenvolvedor", Denoising bullet: when finished, the block is
 * committed to the KV cache and the next one starts).
 * For each layer l, sequence b, kv head g, row t < C:
 *   k_cache[l][b, g, cache_len[b] + t, :] = k_blk[l][(b*C + t)*ld_blk + g*hd ...]
 * (same for v), then cache_len[b] += C.  Tables k_blk, v_blk, k_cache,
 * v_cache are host arrays of n_layers device pointers (n_layers <= 64);
 * hd is 64 or 128 (DG_ERR_UNSUPPORTED_SHAPE otherwise).  A sequence with
 * cache_len[b] + C > lmax is skipped and the device error word records
 * DG_ERR_DEVICE_CHECK.
 */
int dg_kv_block_commit(const void* const* k_blk, const void* const* v_blk, int ld_blk,
                       void* const* k_cache, void* const* v_cache, int32_t* cache_len,
                       int n_layers, int B, int Hkv, int C, int hd, int lmax, void* stream);

/*
 * dg_prefill - causal pass of prompts [B, P] (device int32) through the
 * model; writes their K/V to cache rows [0, P) and sets cache_len to P
 * (and st->cache_len_host).
 * Source: "DiffusionGemma Guia do Desenvolvedor ...", section "Block
 * Autoregressive Diffusion para Sequencias Longas", the Prefill bullet (the
 * prompt is processed with ordinary causal attention and its keys and values
 * go to the KV cache); aiexpert.news architecture paragraph (the same prefill
 * machinery as an autoregressive model); Google docs page "DiffusionGemma",
 * bullet "Arquitetura de codificador-decodificador" (an autoregressive
 * encoder caches the context).  Workspace: dg_prefill_workspace_bytes().
 */
int dg_prefill(const dg_model* m, dg_state* st, const int32_t* prompt, int P,
               void* workspace, size_t workspace_bytes, void* stream);
size_t dg_prefill_workspace_bytes(const dg_model_cfg* cfg, int B, int P);

/*
 * dg_denoise_logits - one bidirectional forward of the current canvas
 * (embedding, layers, final norm, unembedding) over the cached prefix, into
 * logits fp32 [B, C, V].  The building block of dg_denoise_block, exposed for
 * parity tests; with the model's e4m3 unembedding set, the logits are those of
 * the FP8 path (hidden states quantised per token).  Workspace:
 * dg_denoise_block_workspace_bytes().
 */
int dg_denoise_logits(const dg_model* m, const dg_state* st, float* logits,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * dg_denoise_block - denoise one canvas per sequence to its adaptive stop,
 * re-encode it causally and commit its K/V (cache_len += C).
 * Source: "DiffusionGemma Guia do Desenvolvedor ...", section "Block
 * Autoregressive Diffusion para Sequencias Longas", the Denoising bullet (a
 * 256-token block is refined in parallel by bidirectional attention over the
 * cached prefix and, once finished, committed to the KV cache before the next
 * block starts) and section "Difusao de Estado Uniforme" (the block starts
 * as random placeholder tokens); Google docs page "DiffusionGemma", table
 * "Configuracao de exibicao recomendada" (48-step cap, linear 0.8 -> 0.4
 * temperature, adaptive stop on mean entropy below 0.005 with two identical
 * consecutive predictions).  The committed K/V are those of a causal pass
 * over the finished block, so a block-committed cache equals a one-shot
 * causal prefill of the same tokens.
 * Initialises the canvas with uniform tokens (Philox tag 2, counter
 * (0, pos | 2 << 24, 0, block)), runs sampler steps until every sequence has
 * stopped (dg_sample_commit semantics), then the causal re-encode and the
 * block commit.  Synchronises `stream` once per step to read the stop state.
 * Steps after the first replay a CUDA graph of one step's launches, captured
 * on a private stream of the library (set DG_GRAPHS=0 in the environment to
 * launch every step directly; a stream that is itself being captured always
 * gets direct launches).
 * steps_taken (host, may be NULL) receives the largest step count over the batch.
 * Workspace: dg_denoise_block_workspace_bytes().
 */
int dg_denoise_block(const dg_model* m, dg_state* st, const dg_sampler_cfg* cfg, uint32_t seed,
                     int block, int* steps_taken, void* workspace, size_t workspace_bytes,
                     void* stream);
size_t dg_denoise_block_workspace_bytes(const dg_model_cfg* cfg, int B, int C, int lmax);

/*
 * dg_philox4x32_10 - n independent Philox4x32-10 blocks (Salmon et al., SC'11),
 * exposed so that the device generator can be checked against known answers.
 * in: device uint32 [n, 6] = counter words c0..c3 then key words k0, k1;
 * out: device uint32 [n, 4].
 */
int dg_philox4x32_10(const uint32_t* in, uint32_t* out, int n, void* stream);

/*
 * Failure detection.  The pages have no counterpart: these serve the
 * library's own fault handling.  Every wait inside the kernels (on an
 * mbarrier, a CTA-pair barrier or a counter) polls a clock and gives up once
 * it has waited longer than the device's wait limit; it then records
 * DG_ERR_TIMEOUT in the device error word, releases the kernel's other roles
 * and returns, so a lost arrival never hangs the GPU.
 *
 * dg_set_wait_limit_ns - set the wait limit of the current device, in ns
 *   (1 us .. 600 s; 0 restores the default of 2 s).  Enqueued on `stream`,
 *   which it then synchronises; kernels launched afterwards use the new limit.
 * dg_self_test_wait - launch a tiny kernel that waits on an mbarrier nothing
 *   arrives at: kind 0 one CTA (the single-CTA pipeline wait), kind 1 a
 *   cluster of two CTAs (the CTA-pair wait, which also raises the peer's abort
 *   flag).  After it, dg_check_device_errors() returns DG_ERR_TIMEOUT; with a
 *   short limit set first that takes about the limit.  Nothing traps and the
 *   context stays usable.
 */
int dg_set_wait_limit_ns(uint64_t ns, void* stream);
int dg_self_test_wait(int kind, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */

/* dlm.h -- C ABI of libdlm.so: residual block-diffusion decoding at batch size 1 on one
 * B200 (sm_100a).
 *
 * What the library computes (sources cited by page title and section):
 *   - Block-wise diffusion decoding: a block of B masked positions is refined by denoising
 *     rounds; each round yields a distribution over the still-unresolved positions and the
 *     block commits after enough rounds.  ["ORL: diffusion LLMs get a learnable 'tokens per
 *     forward'" (richland.au blog), "What shipped", opening paragraph]
 *   - Residual self-conditioning: the previous round's distribution P_prev is fed back
 *     through an adapter on the tied embedding E.  This library fixes the adapter as
 *     h0_i = E[x_i] + W_a (P_prev,i E), W_a of size d x d.  [same page, "What shipped",
 *     "On-policy residual learning"]
 *   - Block-diffusion attention: block queries attend causally to a prefix KV cache and
 *     bidirectionally within the block (GQA, bf16 KV).  [model card "QwenDLM-4B-ORL"
 *     (shadowgraph.io), "The paper's evaluation pipeline": --dllm-algorithm SDARPrefixKV]
 *   - LM head fused with per-row statistics (max, argmax, logsumexp, max-prob, entropy)
 *     so that logits are not a kernel output.  [same card and section:
 *     SDAR_FUSED_ROW_STATS=1]
 *   - Confidence-threshold commit: positions whose max-prob >= tau commit, at least the
 *     single most confident one per round; a fixed top-k schedule is also offered.
 *     [blog, "What shipped", "Adjacent entropy contraction": "more positions clear the
 *     commit bar"; card: SDAR_COMMIT_GRAPH=1]
 *   - One CUDA graph per block whose conditional (while) node decides after every round
 *     whether to continue, so the host only launches the block and reads tokens back.
 *     [blog, "What shipped", "dlmrt, the inference engine"]
 *
 * Conventions
 *   - Every function returns a dlm_status (0 = DLM_OK), throws nothing and never exits.
 *   - Device pointers are marked d_, host pointers h_.  The caller owns all memory:
 *     weights, workspace, KV cache and block state.  The library keeps pointers only and
 *     never allocates device memory.
 *   - All device work is ordered on the stream passed in (cudaStream_t, passed as void*
 *     so this header needs no CUDA include).  Only dlm_generate synchronizes.
 *   - A context is not thread-safe.  Weights are read-only.
 *   - Matrices are row-major bf16 "out x in" (PyTorch nn.Linear layout) unless stated.
 */
#ifndef DLM_H_
#define DLM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int dlm_status;
#define DLM_OK 0
#define DLM_EINVAL 1        /* null pointer, bad dims, tau NaN, B outside [1,64], k < 1 */
#define DLM_ENOMEM_WS 2     /* workspace or scratch too small */
#define DLM_EKVCAP 3        /* L + B exceeds the KV capacity (max_ctx) */
#define DLM_ECUDA 4         /* a CUDA runtime/driver error; see dlm_last_error */
#define DLM_EROUNDCAP 5     /* a block reached B rounds with positions uncommitted */
#define DLM_ETIMEOUT 6      /* a device-side bounded wait gave up (kernel returned early) */
#define DLM_EUNSUPPORTED 7  /* shape or format the library does not handle */

#define DLM_COMMIT_THRESHOLD 0 /* commit max-prob >= tau, at least one per round */
#define DLM_COMMIT_TOPK 1      /* commit the top min(k, remaining) by max-prob */

#define DLM_FILL_EAGER 0    /* a block's KV-fill forward runs as soon as the block commits */
#define DLM_FILL_DEFERRED 1 /* it is carried by the next round (default; see dlm_kv_fill) */

#define DLM_KV_BF16 0 /* K/V cache rows in bf16 */
#define DLM_KV_FP8 1  /* e4m3 K/V rows, one fp32 scale amax / 448 per row (see dlm_kv_cache_size) */

#define DLM_WEIGHTS_BF16 0
#define DLM_WEIGHTS_NVFP4 1 /* MLP and LM head in NVFP4, attention projections bf16 */

typedef struct dlm_config {
  int n_layers;    /* transformer layers */
  int d;           /* model width; multiple of 64 */
  int n_q_heads;   /* query heads */
  int n_kv_heads;  /* key/value heads; divides n_q_heads */
  int head_dim;    /* 32, 64 or 128 */
  int ffn;         /* SiLU-gated MLP width; multiple of 64 */
  int vocab;       /* V; rows of the tied embedding */
  int mask_id;     /* id of the mask token (embedded by its row of E, never predicted) */
  int max_ctx;     /* KV capacity in positions */
  int block_size;  /* B, in [1, 64] */
  float rope_theta;/* RoPE base (NeoX rotate-half pairing (j, j + hd/2)) */
  float rms_eps;   /* RMSNorm epsilon */
  int weight_fmt;  /* DLM_WEIGHTS_BF16 or DLM_WEIGHTS_NVFP4 */
  int kv_fmt;      /* DLM_KV_BF16 or DLM_KV_FP8 */
} dlm_config;

/* One NVFP4 matrix [rows][cols]: e2m1 codes (2 per byte, element 2j in the low nibble),
 * one e4m3 scale per 16 consecutive elements of a row, and one fp32 tensor scale.
 * Produced by dlm_nvfp4_quantize. */
typedef struct dlm_nvfp4_matrix {
  const void* codes;   /* device, uint8 [rows][cols/2] */
  const void* scales;  /* device, uint8 [rows][cols/16] */
  float tensor_scale;
} dlm_nvfp4_matrix;

typedef struct dlm_layer_weights {
  const void* attn_norm; /* bf16 [d] */
  const void* w_qkv;     /* bf16 [(Hq + 2 Hkv) hd][d]; rows: q heads, k heads, v heads */
  const void* w_o;       /* bf16 [d][Hq hd] */
  const void* mlp_norm;  /* bf16 [d] */
  const void* w_gate;    /* bf16 [F][d] */
  const void* w_up;      /* bf16 [F][d] */
  const void* w_down;    /* bf16 [d][F] */
  dlm_nvfp4_matrix q_gate, q_up, q_down; /* used when weight_fmt == DLM_WEIGHTS_NVFP4 */
} dlm_layer_weights;

typedef struct dlm_weights {
  const void* embed;      /* E, bf16 [V][d]: token embedding and tied LM head (bf16 weights;
                             unused with NVFP4 weights, where E is q_embed throughout) */
  const void* w_adapter;  /* W_a, bf16 [d][d] */
  const void* final_norm; /* bf16 [d] */
  const dlm_layer_weights* layers; /* host array [n_layers]; copied by dlm_ctx_create */
  dlm_nvfp4_matrix q_embed; /* NVFP4 E when weight_fmt == NVFP4: the LM head streams it; the
                               embedding rows and P E use its dequantised values, read from the
                               codes (the workspace holds a bf16 copy, V x d x 2 bytes, only
                               where the LM head runs unfused: B > 32 or d % 512 != 0) */
} dlm_weights;

/* Per-row statistics of one round, device arrays of length B. */
typedef struct dlm_row_stats {
  float* m;        /* max logit */
  float* lse;      /* log-sum-exp */
  float* maxprob;  /* exp(m - lse) */
  float* entropy;  /* nats */
  int32_t* argmax; /* lowest id among the maxima; the mask id is excluded */
} dlm_row_stats;

/* Caller-owned device state of one block (resumable: everything lives here). */
typedef struct dlm_block_state {
  int32_t* tokens;     /* [B]: mask_id or the committed id */
  uint8_t* committed;  /* [B]: 0/1 */
  float* s;            /* [B][d]: residual input P_prev E (zero rows where there is none) */
  int32_t* round;      /* [1]: rounds done in this block */
  int32_t* status;     /* [1]: 0 or a DLM_E* code raised on the device */
  dlm_row_stats stats; /* written by every round */
} dlm_block_state;

typedef struct dlm_timing {
  double prefill_ms;   /* prompt prefill */
  double decode_ms;    /* all blocks, including KV-fill and per-block read-back */
  int n_blocks;
  int n_rounds;        /* denoising rounds in total */
} dlm_timing;

typedef struct dlm_ctx dlm_ctx;

/* ---------------------------------------------------------------- context */
/* Bytes of device workspace a context needs (256-byte aligned base). */
size_t dlm_workspace_size(const dlm_config* cfg);
/* Bytes of the KV cache.  DLM_KV_BF16: values bf16 [layer][K|V][kv_head][max_ctx][head_dim].
 * DLM_KV_FP8 ("ORL: diffusion LLMs get a learnable 'tokens per forward'", "What shipped",
 * "dlmrt, the inference engine": the KV cache is FP8): values e4m3 bytes in the same layout,
 * followed by fp32 scales [layer][K|V][kv_head][max_ctx], one per row of head_dim values:
 * scale = amax(|row|) / 448, value = e4m3(code) * scale (K after RoPE). */
size_t dlm_kv_cache_size(const dlm_config* cfg);
/* Validates cfg, copies the weight pointer table, carves the workspace.  The KV cache
 * layout is [layer][K|V][kv_head][max_ctx][head_dim] bf16.  Sets the prefix length L = 0. */
dlm_status dlm_ctx_create(const dlm_config* cfg, const dlm_weights* w, void* d_workspace,
                          size_t ws_bytes, void* d_kv_cache, size_t kv_bytes, dlm_ctx** out);
dlm_status dlm_ctx_destroy(dlm_ctx* ctx);
/* Message of the last error on this context ("" if none); valid until the next call. */
const char* dlm_last_error(const dlm_ctx* ctx);
/* Current prefix length L (positions of the KV cache holding committed context). */
int dlm_prefix_len(const dlm_ctx* ctx);
/* Sets L (0 <= L <= max_ctx - B).  Rows >= L of the KV cache are treated as free.  A pending
 * KV-fill (see dlm_kv_fill) whose rows lie at or above the new L is dropped; otherwise it is
 * run first. */
dlm_status dlm_set_prefix_len(dlm_ctx* ctx, int L, void* stream);

/* ---------------------------------------------------------------- decoding */
/* Causal prefill of n prompt tokens at positions [L, L + n); L += n.  d_tokens int32 [n]. */
dlm_status dlm_prefill(dlm_ctx* ctx, const int32_t* d_tokens, int n, void* stream);

/* Initialises a block state: tokens = mask_id, committed = 0, s = 0, round = 0, status = 0. */
dlm_status dlm_block_init(dlm_ctx* ctx, const dlm_block_state* st, void* stream);

/* One denoising round over the block at prefix length L (L unchanged), updating the
 * caller's state in place: embedding + residual adapter, the transformer layers with
 * block-diffusion attention (block K/V written to cache rows [L, L+B)), fused LM head
 * with row statistics and s = softmax(logits) E, then the commit rule.  tau is used by
 * DLM_COMMIT_THRESHOLD, tpf_k by DLM_COMMIT_TOPK.  If a KV-fill is pending, this round
 * computes it in the same pass (see dlm_kv_fill). */
dlm_status dlm_round(dlm_ctx* ctx, const dlm_block_state* st, float tau, int commit_mode,
                     int tpf_k, void* stream);
/*   [blog "ORL: diffusion LLMs get a learnable 'tokens per forward'", "What shipped": a
 *   round predicts the still-unresolved positions and feeds its distribution back through
 *   the tied embedding ("On-policy residual learning"); card "QwenDLM-4B-ORL", "The paper's
 *   evaluation pipeline": SDARPrefixKV attention, SDAR_FUSED_ROW_STATS, SDAR_COMMIT_GRAPH] */

/* Clean forward of a committed block (s = 0, no LM head) writing its K/V to rows
 * [L, L+B); then L += B.  d_tokens int32 [B].
 * In DLM_FILL_DEFERRED mode (the default, on contexts with bf16 weights, B <= 32 and the
 * fused LM head) the call only records the block as pending: the next dlm_round (or the
 * next block's graph) prepends the pending block's B rows to its own B rows and computes
 * both in one pass over the weights; the pending rows see the prefix and their own block,
 * the new rows see everything, so the K/V rows written are those of the separate forward
 * (up to fp32 summation order).  Until then rows [L - B, L) of the cache are not valid:
 * dlm_kv_flush writes them.  Other contexts run the forward at once. */
dlm_status dlm_kv_fill(dlm_ctx* ctx, const int32_t* d_tokens, void* stream);

/* Runs a pending KV-fill on its own (no-op if none is pending). */
dlm_status dlm_kv_flush(dlm_ctx* ctx, void* stream);
/* 1 if a KV-fill is pending, 0 if not, -1 for a null context. */
int dlm_fill_pending(const dlm_ctx* ctx);
/* DLM_FILL_EAGER or DLM_FILL_DEFERRED (switching to eager runs a pending fill first). */
dlm_status dlm_set_fill_mode(dlm_ctx* ctx, int mode, void* stream);

/* Decodes one whole block on the device: one launch of a CUDA graph that initialises
 * the block, loops rounds in a while-conditional node until every position is committed
 * (or B rounds), then runs the block's KV-fill.  Writes d_tokens_out int32 [B] and
 * d_rounds_out int32 [2] = {rounds, device status}.  L += B (host and device).  In
 * DLM_FILL_DEFERRED mode the KV-fill is left pending (see dlm_kv_fill) and the next block's
 * graph carries it in its first round: one weight stream per block less.  The graph is
 * instantiated on first use per (commit mode, tau, k, fill variant) and reused. */
dlm_status dlm_decode_block(dlm_ctx* ctx, float tau, int commit_mode, int tpf_k,
                            int32_t* d_tokens_out, int32_t* d_rounds_out, void* stream);
/*   [blog, "What shipped", "dlmrt, the inference engine": one CUDA graph per block with a
 *   conditional node deciding after each round whether to go on; the host launches the
 *   block and reads back tokens] */

/* Host-level generation: copies the prompt to the device, prefills it at L = 0, decodes
 * ceil(max_new / B) blocks with dlm_decode_block, reading each block's tokens back, runs the
 * last block's pending KV-fill (the cache holds every block on return), and returns max_new
 * tokens (the last block truncated) and the rounds of every block.
 * Synchronizes.  h_prompt int32 [prompt_len]; h_tokens_out int32 [max_new];
 * h_rounds_per_block int32 [ceil(max_new/B)] (may be NULL); h_timing may be NULL. */
dlm_status dlm_generate(dlm_ctx* ctx, const int32_t* h_prompt, int prompt_len, int max_new,
                        float tau, int commit_mode, int tpf_k, int32_t* h_tokens_out,
                        int32_t* h_rounds_per_block, dlm_timing* h_timing, void* stream);
/*   [card "QwenDLM-4B-ORL", usage section: generate(prompt, max_new_tokens) on one request;
 *   blog, "What shipped": block-wise decoding over a prefix KV cache] */

/* ---------------------------------------------------------------- single operations
 * Stand-alone entry points of the kernels one round is made of, used by the parity tests
 * and the per-kernel benchmarks.  `scratch` is caller-owned device memory of at least
 * the size the matching *_scratch_size function returns. */

/* y[T][N] (fp32) = x[T][K] (bf16) W[N][K]^T (bf16) on the tensor cores.  T <= 256,
 * K % 8 == 0, K >= 64.  d_y may be NULL: then only the tensor-core kernel runs and its
 * fp32 partial sums stay in the scratch (used to time that kernel alone). */
size_t dlm_gemm_scratch_size(int T, int N, int K);
dlm_status dlm_gemm_bf16(const void* d_x, const void* d_w, float* d_y, int T, int N, int K,
                         void* d_scratch, size_t scratch_bytes, void* stream);

/* The same GEMM with split activations, the form every projection of a round uses:
 * x = hi + lo, both bf16, so the activations carry about 16 significant bits while the
 * weight tile is still streamed from HBM once.  d_x2 holds 2 * dlm_split_pad(T) rows of K:
 * high halves in rows [0, T), low halves in rows [pad, pad + T).  T <= 128. */
int dlm_split_pad(int T);
dlm_status dlm_gemm_bf16x2(const void* d_x2, const void* d_w, float* d_y, int T, int N, int K,
                           void* d_scratch, size_t scratch_bytes, void* stream);

/* The same GEMM taking fp32 activations x[T][K]: the library splits them into the
 * hi + lo bf16 pair itself (in the scratch) and runs dlm_gemm_bf16x2.  T <= 128. */
size_t dlm_gemm_f32_scratch_size(int T, int N, int K);
dlm_status dlm_gemm_f32(const float* d_x, const void* d_w, float* d_y, int T, int N, int K,
                        void* d_scratch, size_t scratch_bytes, void* stream);

/* LM head fused with row statistics and the residual contraction:
 *   logits = x E^T (x: bf16 [B][d], already normalised), stats of every row with the
 *   mask id excluded (mask_id < 0: none excluded), and s = P E with P = softmax(logits)
 *   (d_p_given == NULL; P carried as a split bf16 pair) or P = d_p_given (bf16 [B][V]).
 *   s: fp32 [B][d].  B <= 128. */
size_t dlm_lmhead_scratch_size(int B, int V, int d);
dlm_status dlm_lmhead_rowstats(const void* d_x, const void* d_embed, int B, int V, int d,
                               int mask_id, const void* d_p_given, dlm_row_stats stats,
                               float* d_s, void* d_scratch, size_t scratch_bytes, void* stream);

/* Adapter step: h0[B][d] (fp32) = E[tokens] + W_a s, s fp32 [B][d] (carried into the GEMM
 * as a split bf16 pair).  B <= 128. */
size_t dlm_adapter_scratch_size(int B, int d);
dlm_status dlm_adapter_embed(const void* d_embed, const void* d_w_adapter, const int32_t* d_tokens,
                             const float* d_s, float* d_h0, int B, int d, void* d_scratch,
                             size_t scratch_bytes, void* stream);

/* Block-diffusion attention of one layer: T queries at positions [L, L+T) against the
 * cache rows [0, L+T) of one layer (causal != 0: query at position p sees keys [0, p]).
 * q bf16 [T][Hq][hd]; k_cache, v_cache bf16 [Hkv][max_ctx][hd]; o bf16 [T][Hq][hd]. */
size_t dlm_attention_scratch_size(int T, int Hq, int hd, int max_ctx);
dlm_status dlm_bd_attention(const void* d_q, const void* d_k_cache, const void* d_v_cache,
                            void* d_o, int T, int L, int Hq, int Hkv, int hd, int max_ctx,
                            int causal, void* d_scratch, size_t scratch_bytes, void* stream);

/* The same attention with no scratch argument, for callers that cannot give the library
 * device memory beyond the operands (nothing is allocated by the call).  The pages have no
 * counterpart: it is an interface variant of dlm_bd_attention.  Its split-KV partials live
 * in a fixed 16 MiB array of static device memory per device; calls whose partials
 * (split count x T x Hq x (hd + 2) x 4 bytes, the split count as dlm_bd_attention picks it
 * from T, Hq, Hkv and max_ctx) exceed 16 MiB - 256 B are rejected with DLM_ENOMEM_WS.  The
 * 4B-class shapes (T <= 64, 32/8 heads, hd 128) need at most 9.9 MB.  The first call on
 * each device looks the array up and sets the kernels' attributes on that device: make it
 * before starting any stream capture on that device.  A call launches the attention kernels
 * only (the partials need no clearing).  The array is shared: calls that may overlap in
 * time race on it and must be serialised by the caller. */
dlm_status dlm_bd_attention_noalloc(const void* d_q, const void* d_k_cache, const void* d_v_cache,
                                    void* d_o, int T, int L, int Hq, int Hkv, int hd, int max_ctx,
                                    int causal, void* stream);

/* One layer's MLP sub-block on given residual rows (single operation for parity tests):
 * h_out = h_in + W_down (silu(W_gate x) * (W_up x)), x = RMSNorm(h_in) g_mlp, with the
 * context's weights of that layer (for NVFP4 weights x and the SiLU output are quantized per
 * row, as in a round).  d_h_in, d_h_out fp32 [T][d]; T <= 64 (NVFP4) or <= 128.  Uses the
 * context's workspace: not concurrent with other calls on the context. */
dlm_status dlm_mlp_block(dlm_ctx* ctx, int layer, const float* d_h_in, float* d_h_out, int T, void* stream);

/* The same attention on an FP8 KV cache (see dlm_kv_cache_size): k_codes, v_codes uint8
 * [Hkv][max_ctx][hd] e4m3; k_scales, v_scales fp32 [Hkv][max_ctx].  The e4m3 values enter
 * the tensor cores exactly (as bf16); the K row scales multiply the scores and the V row
 * scales the softmax weights.  Scratch as dlm_bd_attention. */
dlm_status dlm_bd_attention_fp8(const void* d_q, const void* d_k_codes, const float* d_k_scales,
                                const void* d_v_codes, const float* d_v_scales, void* d_o, int T, int L,
                                int Hq, int Hkv, int hd, int max_ctx, int causal, void* d_scratch,
                                size_t scratch_bytes, void* stream);

/* Commit rule on device arrays (one block of B positions).  Updates tokens, committed,
 * zeroes the s rows of newly committed positions, increments *d_round. */
dlm_status dlm_commit(const float* d_maxprob, const int32_t* d_argmax, int32_t* d_tokens,
                      uint8_t* d_committed, float* d_s, int32_t* d_round, int32_t* d_status,
                      int B, int d, float tau, int commit_mode, int tpf_k, void* stream);

/* NVFP4 quantizer (per-tensor fp32 scale amax / (6 * 448), e4m3 scale per 16 elements,
 * round-to-nearest-even e2m1 codes) of a bf16 [rows][cols] matrix, cols % 16 == 0.
 * Writes codes uint8 [rows][cols/2], scales uint8 [rows][cols/16], *d_tensor_scale. */
dlm_status dlm_nvfp4_quantize(const void* d_w, int rows, int cols, void* d_codes, void* d_scales,
                              float* d_tensor_scale, void* stream);

/* NVFP4 weight GEMM: y[T][N] (fp32) = Q(x) W^T, where W is an NVFP4 matrix [N][K] (see
 * dlm_nvfp4_matrix; host struct, device arrays) and Q(x) quantizes each row of x (fp32
 * [T][K]) to NVFP4 with its own fp32 scale amax_row / (6 * 448), e4m3 scales per 16 elements
 * and round-to-nearest-even e2m1 codes, the format the pages' B200 numbers use ("ORL:
 * diffusion LLMs get a learnable 'tokens per forward'", "What shipped"), on the
 * block-scaled FP4 tensor cores.  T <= 64, K % 256 == 0, K <= 16384.  d_y may be NULL:
 * partial sums only (kernel timing). */
size_t dlm_gemm_nvfp4_scratch_size(int T, int N, int K);
dlm_status dlm_gemm_nvfp4(const float* d_x, const dlm_nvfp4_matrix* w, float* d_y, int T, int N, int K,
                          void* d_scratch, size_t scratch_bytes, void* stream);

/* The fused LM head of dlm_lmhead_rowstats with an NVFP4 embedding E [V][d] (see
 * dlm_nvfp4_matrix; host struct, device arrays): x (fp32 [B][d], already normalised) is
 * quantized per row as for dlm_gemm_nvfp4, the logits S_E S_x[t] (q_x sigma_x)(q_E sigma_E)^T
 * run on the block-scaled FP4 tensor cores and are never stored, and s = P E uses the
 * dequantized E (e2m1 x e4m3 values, exact in f16) with P = softmax(logits) carried as f16,
 * in the same pass over E ("QwenDLM-4B-ORL" model card, "The paper's evaluation pipeline": the
 * LM head with fused row statistics; "ORL: diffusion LLMs get a learnable 'tokens per
 * forward'", "What shipped": NVFP4 weights).  Mask id as dlm_lmhead_rowstats.  B <= 32,
 * d % 512 == 0, d <= 2560; other shapes return DLM_EUNSUPPORTED (scratch size 0). */
size_t dlm_lmhead_nvfp4_scratch_size(int B, int V, int d);
dlm_status dlm_lmhead_rowstats_nvfp4(const float* d_x, const dlm_nvfp4_matrix* E, int B, int V, int d, int mask_id,
                                     dlm_row_stats stats, float* d_s, void* d_scratch, size_t scratch_bytes,
                                     void* stream);

/* Routed-expert MLP sub-block with NVFP4 experts ([blog] "ORL: diffusion LLMs get a learnable
 * 'tokens per forward'", "What shipped", "dlmrt, the inference engine": routed experts run
 * NVFP4 on FP4 tensor cores).  The pages give neither the routing rule nor the expert shapes;
 * the library's reading:
 *   x = RMSNorm(h) g;  l = x W_r^T;  the k experts of largest l (ties to the lower index),
 *   weighted by softmax renormalised over the chosen: w_e = exp(l_e) / sum_chosen exp(l_j);
 *   h_out = h + sum_e w_e down_e(silu(gate_e x) * (up_e x)).
 * The E experts' gate and up matrices are stacked along rows ([E F][d], expert e in rows
 * [e F, (e + 1) F)) and their down matrices side by side along columns ([d][E F]), each stack
 * one NVFP4 matrix (see dlm_nvfp4_matrix).  x is quantized per row for the gate/up GEMM; the
 * activation row entering the down projection is the concatenation over the experts of
 * w_e silu(.) * up(.) (zeros for the experts not chosen), quantized per row, so the weighted
 * sum over the experts is one FP4 contraction over E F.  Every expert's weights are streamed
 * (at 32 rows and k of E experts most experts are chosen by some row). */
typedef struct dlm_moe_weights {
  int n_experts;      /* E, 1..256 */
  int top_k;          /* k, 1..min(E, 8) */
  int ffn_expert;     /* F, a multiple of 64; E F a multiple of 256 */
  const void* w_router;   /* device, bf16 [E][d] */
  const void* mlp_norm;   /* device, bf16 [d] */
  dlm_nvfp4_matrix q_gate, q_up;  /* [E F][d] */
  dlm_nvfp4_matrix q_down;        /* [d][E F] */
} dlm_moe_weights;

/* The experts' e4m3 scales re-tiled for the block-scaled MMA (done once per weight set):
 * d_tiles receives dlm_moe_prepare_size(d, w) bytes. */
size_t dlm_moe_prepare_size(int d, const dlm_moe_weights* w);
dlm_status dlm_moe_prepare(int d, const dlm_moe_weights* w, void* d_tiles, size_t bytes, void* stream);

/* One sub-block on T <= 64 rows: h_in, h_out fp32 [T][d] (distinct buffers), d % 256 == 0,
 * d <= 8192; d_tiles from dlm_moe_prepare.  Outputs the chosen experts (int32 [T][k]) and their
 * weights (fp32 [T][k]) when the pointers are non-null.  Scratch: dlm_moe_scratch_size bytes,
 * DLM_ENOMEM_WS if smaller; DLM_EUNSUPPORTED for shapes outside the limits. */
size_t dlm_moe_scratch_size(int T, int d, const dlm_moe_weights* w);
dlm_status dlm_moe_mlp_nvfp4(const float* d_h_in, float* d_h_out, int T, int d, float rms_eps,
                             const dlm_moe_weights* w, const void* d_tiles, int32_t* d_topk_idx,
                             float* d_topk_w, void* d_scratch, size_t scratch_bytes, void* stream);

/* Version string of the build. */
const char* dlm_version(void);

/* Debugging aid: 1 (default) launches the kernels of a round with programmatic dependent
 * launch (each kernel starts while its predecessor drains; weight tiles are prefetched
 * before the dependency resolves), 0 launches them plainly stream-ordered. */
void dlm_debug_set_pdl(int on);

#ifdef __cplusplus
}
#endif

#endif /* DLM_H_ */

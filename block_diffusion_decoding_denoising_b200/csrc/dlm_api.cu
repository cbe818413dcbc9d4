// dlm_api.cu -- context, workspace layout, round orchestration, the per-block CUDA graph
// and the extern "C" entry points of libdlm.so (declared in include/dlm.h).
//
// The per-block graph ["ORL: diffusion LLMs get a learnable 'tokens per forward'"
// (richland.au blog), "What shipped", "dlmrt, the inference engine": the denoising loop
// of a block stays on the GPU and a conditional node decides after every round whether
// to continue]:
//
//   [init: tokens = MASK, committed = 0, s = 0, round = 0]
//     -> WHILE(cond) { one denoising round ... k_commit sets cond = any uncommitted
//                      && round < B through cudaGraphSetConditional }
//     -> [KV-fill forward of the committed block, L += B, copy tokens/rounds out]
//
// The prefix length L lives in device memory (ctx->d_L) so the same instantiated graph
// serves every block; the host keeps a mirror for argument checks.
#include <chrono>
#include <new>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "dlm_internal.h"
#include "dlm_ops.h"

using namespace dlm;

namespace {

constexpr int kPrefillChunk = kMaxSplitTokens;  // prefill tokens per forward pass (bf16 weights)
constexpr int kRowChunk = 4096;                  // vocabulary entries per row-statistics CTA

// Per-block graph variants: the KV-fill of the block runs inside its own graph (EAGER), or
// is left pending and carried by the first round of the next block (FIRST: no block pending
// at launch, FOLD: one pending block folded into the first round).
enum GraphVariant : int { GV_EAGER = 0, GV_FIRST = 1, GV_FOLD = 2 };

struct GraphEntry {
  int mode;
  float tau;
  int k;
  int variant;
  cudaGraph_t graph;
  cudaGraphExec_t exec;
};

}  // namespace

struct dlm_ctx {
  dlm_config cfg;
  dlm_weights w;
  std::vector<dlm_layer_weights> layers;
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  uint8_t* kv = nullptr;   // KV cache values (bf16 or e4m3), then for FP8 the row scales
  size_t kv_bytes = 0;
  int L = 0;
  int Tmax = 0;
  // workspace carve
  int* d_L = nullptr;
  int* d_err = nullptr;
  float* h = nullptr;
  __nv_bfloat16* xn = nullptr;
  __nv_bfloat16* q = nullptr;
  __nv_bfloat16* o = nullptr;
  __nv_bfloat16* act = nullptr;
  __nv_bfloat16* sbf = nullptr;
  float* partial = nullptr;
  size_t partial_bytes = 0;
  int* tile_cnt = nullptr;   // per-tile arrival counters of the GEMM epilogue
  float* ss = nullptr;       // per-tile sums of squares [ceil(d/128)][Tmax]
  float* rs_part = nullptr;  // row-statistics chunk partials
  float2* rope_tab = nullptr;  // [max_ctx][hd/2] (cos, sin)
  float* attn_part = nullptr;
  int attn_splits_B = 1, attn_splits_T = 1, attn_splits_2B = 1;
  // deferred KV-fill: a committed block whose clean forward has not run yet (its K/V rows
  // [L - B, L) are not valid); the next round carries it, dlm_kv_flush runs it alone
  int32_t* pend_tokens = nullptr;  // device [B]
  bool pending = false;
  bool fill_deferred = true;       // dlm_set_fill_mode
  float* logits = nullptr;
  __nv_bfloat16* P = nullptr;
  int32_t* tok_buf = nullptr;
  // NVFP4 weights: quantized GEMM inputs, their row scales, and E dequantised to bf16
  // (q sigma, exact; the tensor scale is applied where the rows are used)
  void* lmf = nullptr;  // scratch of the fused LM head (null: the unfused path is used)
  bool fp4 = false;
  uint8_t* xcodes = nullptr;   // [32][max(d, F) / 2] e2m1 codes of the GEMM input
  uint8_t* xscales = nullptr;  // e4m3 scales, tiled [max(d, F) / 64][32][16 B]
  float* sx = nullptr;
  float* act_amax = nullptr;   // [F / 64][Tmax] partial maxima of the SiLU output (NVFP4)
  __nv_bfloat16* e_deq = nullptr;
  uint8_t* sf = nullptr;       // weight scales re-tiled for the FP4 MMA: per layer (gate/up, down), then E
  size_t sf_pair = 0, sf_down = 0;
  // internal block state (graph path)
  int32_t* b_tokens = nullptr;
  uint8_t* b_committed = nullptr;
  float* b_s = nullptr;
  int32_t* b_round = nullptr;
  int32_t* b_status = nullptr;
  dlm_row_stats b_stats{};
  int32_t* out_tokens = nullptr;
  int32_t* out_rounds = nullptr;
  cudaStream_t cap_stream = nullptr;
  std::vector<GraphEntry> graphs;
  std::string err;
};

namespace {

// ------------------------------------------------------------------ helpers
dlm_status fail(dlm_ctx* ctx, dlm_status code, const char* fmt, ...) {
  if (ctx) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    ctx->err = buf;
  }
  return code;
}

#define CU(call)                                                                              \
  do {                                                                                        \
    cudaError_t e_ = (call);                                                                  \
    if (e_ != cudaSuccess)                                                                    \
      return fail(ctx, DLM_ECUDA, "%s:%d %s: %s", __FILE__, __LINE__, #call, cudaGetErrorString(e_)); \
  } while (0)

#define CU_LAUNCH(call) CU(call)

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Carver {
  uint8_t* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    off = align256(off);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

int max_tokens(const dlm_config& c) {
  return c.block_size > kPrefillChunk ? c.block_size : kPrefillChunk;
}

// Tokens per prefill forward: the NVFP4 GEMM takes at most kMaxF4Tokens.
int prefill_chunk(const dlm_config& c) {
  return c.weight_fmt == DLM_WEIGHTS_NVFP4 ? kMaxF4Tokens : kPrefillChunk;
}

size_t max_partial_bytes(const dlm_config& c, int Tmax) {
  const int qkv = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim, ho = c.n_q_heads * c.head_dim;
  size_t m = 0;
  for (int T : {c.block_size, Tmax}) {
    size_t v[] = {gemm_partial_bytes(T, c.d, c.d, A_KMAJOR), gemm_partial_bytes(T, qkv, c.d, A_KMAJOR),
                  gemm_partial_bytes(T, c.d, ho, A_KMAJOR), gemm_partial_bytes(T, c.ffn, c.d, A_PAIR),
                  gemm_partial_bytes(T, c.d, c.ffn, A_KMAJOR)};
    for (size_t x : v) m = x > m ? x : m;
  }
  const int B = c.block_size;
  size_t lm = gemm_partial_bytes(B, c.vocab, c.d, A_KMAJOR);
  size_t pe = gemm_partial_bytes(B, c.d, c.vocab, A_MNMAJOR);
  m = lm > m ? lm : m;
  m = pe > m ? pe : m;
  if (c.weight_fmt == DLM_WEIGHTS_NVFP4 && c.d % 256 == 0 && c.ffn % 256 == 0) {
    for (int T : {c.block_size, kMaxF4Tokens}) {
      size_t v[] = {gemm_fp4_partial_bytes(T, c.ffn, c.d, A_PAIR), gemm_fp4_partial_bytes(T, c.d, c.ffn, A_KMAJOR),
                    gemm_fp4_partial_bytes(T, c.vocab, c.d, A_KMAJOR)};
      for (size_t x : v) m = x > m ? x : m;
    }
  }
  return m;
}

// Lays out the workspace (base == nullptr: size only).
size_t carve(dlm_ctx* x, const dlm_config& c, uint8_t* base) {
  Carver cv{base};
  const int Tmax = max_tokens(c), B = c.block_size, ho = c.n_q_heads * c.head_dim;
  // GEMM inputs are split bf16 pairs: 2 * pad rows (high halves, then low halves)
  const size_t R2 = 2 * (size_t)split_pad(Tmax), B2 = 2 * (size_t)split_pad(B);
  int* hdr = cv.take<int>(64);
  float* h = cv.take<float>((size_t)Tmax * c.d);
  auto* xn = cv.take<__nv_bfloat16>(R2 * c.d);
  auto* q = cv.take<__nv_bfloat16>((size_t)Tmax * ho);
  auto* o = cv.take<__nv_bfloat16>(R2 * ho);
  auto* act = cv.take<__nv_bfloat16>(R2 * c.ffn);
  auto* sbf = cv.take<__nv_bfloat16>(R2 * c.d);  // W_a input of a pass of up to Tmax rows
  size_t pb = max_partial_bytes(c, Tmax);
  float* partial = cv.take<float>(pb / sizeof(float));
  int* cnt = cv.take<int>((size_t)(c.vocab + 63) / 64 + (c.ffn + 63) / 64 + 64);
  float* ssb = cv.take<float>((size_t)((c.d + 127) / 128) * Tmax);
  float* rsp = cv.take<float>((size_t)4 * B * ((c.vocab + kRowChunk - 1) / kRowChunk));
  float2* rtab = cv.take<float2>((size_t)c.max_ctx * (c.head_dim / 2));
  int sB = attention_max_splits(B, c.n_q_heads, c.n_kv_heads, c.max_ctx);
  int sT = attention_max_splits(Tmax, c.n_q_heads, c.n_kv_heads, c.max_ctx);
  int s2 = attention_max_splits(2 * B, c.n_q_heads, c.n_kv_heads, c.max_ctx);
  size_t ab = attention_scratch_bytes(B, c.n_q_heads, c.head_dim, sB);
  size_t at = attention_scratch_bytes(Tmax, c.n_q_heads, c.head_dim, sT);
  size_t a2 = attention_scratch_bytes(2 * B, c.n_q_heads, c.head_dim, s2);
  size_t amax = ab > at ? ab : at;
  amax = a2 > amax ? a2 : amax;
  float* attn = cv.take<float>(amax / sizeof(float));
  float* logits = cv.take<float>((size_t)B * c.vocab);
  auto* P = cv.take<__nv_bfloat16>(B2 * c.vocab);
  int32_t* tok = cv.take<int32_t>((size_t)c.max_ctx);
  int32_t* bt = cv.take<int32_t>(B);
  uint8_t* bc = cv.take<uint8_t>(B);
  float* bs = cv.take<float>((size_t)B * c.d);
  int32_t* br = cv.take<int32_t>(4);
  float* st = cv.take<float>((size_t)4 * B);
  int32_t* sa = cv.take<int32_t>(B);
  int32_t* ot = cv.take<int32_t>(B);
  int32_t* orr = cv.take<int32_t>(4);
  int32_t* pend = cv.take<int32_t>(B);
  const bool fp4 = c.weight_fmt == DLM_WEIGHTS_NVFP4;
  const size_t kmax = c.d > c.ffn ? c.d : c.ffn;
  uint8_t* xcodes = fp4 ? cv.take<uint8_t>((size_t)kMaxF4Tokens * kmax / 2) : nullptr;
  uint8_t* xscales = fp4 ? cv.take<uint8_t>(f4_scale_bytes(kmax)) : nullptr;
  float* sx = fp4 ? cv.take<float>(kMaxF4Tokens) : nullptr;
  float* aam = fp4 ? cv.take<float>((size_t)((c.ffn + 63) / 64) * Tmax) : nullptr;
  const bool fp4_shapes = fp4 && c.d % 256 == 0 && c.ffn % 256 == 0;
  const bool fused = fp4 ? fp4_shapes && lmhead_fused_f4_supported(B, c.d) : lmhead_fused_supported(B, c.d);
  // a bf16 copy of the NVFP4 E (q sigma) only for the unfused LM head's P E; the fused one and
  // the embedding rows read the codes
  __nv_bfloat16* edq = (fp4 && !fused) ? cv.take<__nv_bfloat16>((size_t)c.vocab * c.d) : nullptr;
  const size_t sfp = fp4_shapes ? align256(nvf4_sf_tile_bytes(c.ffn, c.d, A_PAIR)) : 0;
  const size_t sfd = fp4_shapes ? align256(nvf4_sf_tile_bytes(c.d, c.ffn, A_KMAJOR)) : 0;
  const size_t sfe = fp4_shapes ? align256(nvf4_sf_tile_bytes(c.vocab, c.d, A_KMAJOR)) : 0;
  uint8_t* sf = fp4_shapes ? cv.take<uint8_t>((size_t)c.n_layers * (sfp + sfd) + sfe) : nullptr;
  uint8_t* lmf = fused ? cv.take<uint8_t>(lmhead_fused_scratch_bytes(c.vocab, c.d)) : nullptr;
  if (x && base) {
    x->lmf = lmf;
    x->fp4 = fp4;
    x->xcodes = xcodes;
    x->xscales = xscales;
    x->sx = sx;
    x->act_amax = aam;
    x->sf = sf;
    x->sf_pair = sfp;
    x->sf_down = sfd;
    x->e_deq = edq;
    x->d_L = hdr;
    x->d_err = hdr + 1;
    x->h = h;
    x->xn = xn;
    x->q = q;
    x->o = o;
    x->act = act;
    x->sbf = sbf;
    x->partial = partial;
    x->partial_bytes = pb;
    x->tile_cnt = cnt;
    x->ss = ssb;
    x->rs_part = rsp;
    x->rope_tab = rtab;
    x->attn_part = attn;
    x->attn_splits_B = sB;
    x->attn_splits_T = sT;
    x->attn_splits_2B = s2;
    x->pend_tokens = pend;
    x->logits = logits;
    x->P = P;
    x->tok_buf = tok;
    x->b_tokens = bt;
    x->b_committed = bc;
    x->b_s = bs;
    x->b_round = br;
    x->b_status = br + 1;
    x->b_stats = dlm_row_stats{st, st + B, st + 2 * B, st + 3 * B, sa};
    x->out_tokens = ot;
    x->out_rounds = orr;
    x->Tmax = Tmax;
  }
  return align256(cv.off);
}

bool valid_cfg(const dlm_config* c, char* msg, size_t n) {
  if (!c) { snprintf(msg, n, "null config"); return false; }
  if (c->n_layers < 0 || c->d < 64 || c->d % 64 || c->d > 4096 || c->n_q_heads < 1 || c->n_kv_heads < 1 ||
      c->n_q_heads % c->n_kv_heads || !(c->head_dim == 32 || c->head_dim == 64 || c->head_dim == 128) ||
      c->ffn < 64 || c->ffn % 64 || c->vocab < 2 || c->vocab % 8 || c->mask_id < 0 ||
      c->mask_id >= c->vocab || c->block_size < 1 || c->block_size > 64 ||
      c->max_ctx < c->block_size || !(c->rms_eps > 0.f) || !(c->rope_theta > 0.f) ||
      (c->n_q_heads * c->head_dim) % 64) {
    snprintf(msg, n, "invalid dlm_config");
    return false;
  }
  if (c->weight_fmt != DLM_WEIGHTS_BF16 && c->weight_fmt != DLM_WEIGHTS_NVFP4) {
    snprintf(msg, n, "invalid weight_fmt %d", c->weight_fmt);
    return false;
  }
  // FP8 cache: the row scales are read in 16-byte groups of 4 (max_ctx a multiple of 4)
  if ((c->kv_fmt != DLM_KV_BF16 && c->kv_fmt != DLM_KV_FP8) || (c->kv_fmt == DLM_KV_FP8 && c->max_ctx % 4)) {
    snprintf(msg, n, "invalid kv_fmt %d (FP8 needs max_ctx %% 4 == 0)", c->kv_fmt);
    return false;
  }
  return true;
}

// ------------------------------------------------------------------ launch helpers
struct Runner {
  dlm_ctx* ctx;
  cudaStream_t s;
  char msg[512];

  // One projection with split activations and the fused epilogue `epi`.
  dlm_status gemm(int a_mode, const void* a0, const void* a1, const void* x, int T, int N, int K,
                  EpiArgs epi, GemmOut* out = nullptr) {
    GemmPlan p;
    if (!gemm_plan(&p, a_mode, a0, a1, x, T, N, K, ctx->partial, msg, sizeof(msg), true))
      return fail(ctx, DLM_EUNSUPPORTED, "%s", msg);
    if (p.partial_bytes > ctx->partial_bytes)
      return fail(ctx, DLM_ENOMEM_WS, "gemm partials %zu > %zu", p.partial_bytes, ctx->partial_bytes);
    epi.tile_cnt = ctx->tile_cnt;
    p.epi = epi;
    cudaError_t e = gemm_launch(p, ctx->d_err, s);
    if (e != cudaSuccess) return fail(ctx, DLM_ECUDA, "gemm launch: %s", cudaGetErrorString(e));
    if (out) *out = p.out;
    return DLM_OK;
  }
  // A projection that leaves per-slot partial sums (finished by the next kernel).
  dlm_status gemm_partial(int a_mode, const void* a0, const void* a1, const void* x, int T, int N, int K,
                          GemmOut* out) {
    EpiArgs e{};
    e.op = EPI_PARTIAL;
    return gemm(a_mode, a0, a1, x, T, N, K, e, out);
  }
  // NVFP4 projection of the quantized activations in ctx->xcodes / xscales (see act_quant);
  // `sfa`: the weight's re-tiled scales.
  dlm_status gemm_fp4(int a_mode, const dlm_nvfp4_matrix& w0, const dlm_nvfp4_matrix* w1, const uint8_t* sfa, int T,
                      int N, int K, GemmOut* out) {
    GemmF4Plan p;
    if (!gemm_fp4_plan(&p, a_mode, w0, w1, sfa, ctx->xcodes, ctx->xscales, kMaxF4Tokens, ctx->sx, T, N, K,
                       ctx->partial, msg, sizeof(msg)))
      return fail(ctx, DLM_EUNSUPPORTED, "%s", msg);
    if (p.partial_bytes > ctx->partial_bytes)
      return fail(ctx, DLM_ENOMEM_WS, "nvfp4 gemm partials %zu > %zu", p.partial_bytes, ctx->partial_bytes);
    cudaError_t e = gemm_fp4_launch(p, ctx->d_err, s);
    if (e != cudaSuccess) return fail(ctx, DLM_ECUDA, "nvfp4 gemm launch: %s", cudaGetErrorString(e));
    *out = p.out;
    return DLM_OK;
  }
  dlm_status check() {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ctx, DLM_ECUDA, "launch: %s", cudaGetErrorString(e));
    return DLM_OK;
  }
};

#define TRY(x)                      \
  do {                              \
    dlm_status st_ = (x);           \
    if (st_ != DLM_OK) return st_;  \
  } while (0)

struct FwdSpec {
  int T;
  const int32_t* tokens;  // device [T]
  // A pending committed block (T_pend = B rows, or 0) computed ahead of the T rows in the same
  // pass: its clean forward (s = 0) at positions [pos - T_pend, pos), each of its rows seeing
  // the prefix and its own block, while the T rows see everything.  Its K/V rows are what a
  // separate KV-fill forward would write; the LM head runs on the T rows only.
  int T_pend;
  const int32_t* pend_tokens;  // device [T_pend]
  const float* s;         // device fp32 [T][d], or nullptr (no adapter)
  int pos0;               // used when !dev_L
  bool dev_L;             // positions from ctx->d_L (graph mode)
  bool causal;
  bool lm_head;           // round: LM head + stats + s_out
  dlm_row_stats stats;
  float* s_out;
};

// h update + RMSNorm into the split GEMM input xn, a 4-CTA cluster per token (see k_resid_norm).
dlm_status resid_norm(Runner& r, int T, const GemmOut* y, const int32_t* embed_tokens, const void* gain,
                      bool quantize = false, const int32_t* embed_tokens2 = nullptr, int tok_split = 0) {
  dlm_ctx* ctx = r.ctx;
  const dlm_config& c = ctx->cfg;
  ResNormArgs a{};
  if (y) a.out = *y;
  a.out.T = T;
  a.h = ctx->h;
  if (embed_tokens && ctx->fp4 && !ctx->e_deq) {  // NVFP4 E read as codes (no bf16 copy kept)
    a.embed_codes = (const uint8_t*)ctx->w.q_embed.codes;
    a.embed_sc = (const uint8_t*)ctx->w.q_embed.scales;
  } else {
    a.embed = embed_tokens ? (ctx->fp4 ? ctx->e_deq : (const __nv_bfloat16*)ctx->w.embed) : nullptr;
  }
  a.tokens = embed_tokens;
  a.tokens2 = embed_tokens2;
  a.tok_split = tok_split;
  a.embed_scale = ctx->fp4 ? ctx->w.q_embed.tensor_scale : 1.0f;
  a.gain = (const __nv_bfloat16*)gain;
  a.xn = ctx->xn;
  a.xn_lo = (long)split_pad(T) * c.d;
  a.d = c.d;
  a.eps = c.rms_eps;
  if (quantize) {  // the next GEMM is NVFP4: quantize its input here (see k_act_quant)
    a.qcodes = ctx->xcodes;
    a.qscales = ctx->xscales;
    a.qsx = ctx->sx;
  }
  CU_LAUNCH(launch_k_cluster(k_resid_norm, dim3(T * kRnCluster), dim3(256), 0, r.s, kRnCluster, a));
  return DLM_OK;
}

// Quantizes the T rows of a split bf16 GEMM input (hi at x, lo at x + lo) to NVFP4 in
// ctx->xcodes / xscales / sx (see k_act_quant).
dlm_status act_quant(Runner& r, int T, const __nv_bfloat16* x, long lo, int K) {
  dlm_ctx* ctx = r.ctx;
  ActQuantArgs a{};
  a.xb = x;
  a.xb_lo = lo;
  a.K = K;
  a.codes = ctx->xcodes;
  a.scales = ctx->xscales;
  a.sx = ctx->sx;
  CU_LAUNCH(launch_k(k_act_quant, dim3(T), dim3(256), 0, r.s, a));
  return DLM_OK;
}

// Finishes the tiles of a partial-sums GEMM with `epi` (one CTA per tile and 32 tokens; the
// plain store one CTA per tile and token).
dlm_status finish_tiles(Runner& r, const GemmOut& y, int N, const EpiArgs& epi) {
  dlm_ctx* ctx = r.ctx;
  FinishArgs a{y, epi, N};
  if (epi.op != EPI_QKV && epi.op != EPI_SILU) {  // one thread per feature and token
    CU_LAUNCH(launch_k(k_finish_store, dim3(y.n_tiles, y.T), dim3(kTileM), 0, r.s, a));
    return DLM_OK;
  }
  void (*k)(FinishArgs) = epi.op == EPI_QKV ? k_finish_qkv : k_finish_silu;
  CU_LAUNCH(launch_k(k, dim3(y.n_tiles, (y.T + 31) / 32), dim3(256), 0, r.s, a));
  return DLM_OK;
}

// The MLP of layer l on the normed input in ctx->xn (and, for NVFP4 weights, its codes):
// gate/up GEMM -> SiLU gate -> [input quantizer ->] down GEMM; the down projection's
// partial sums are left in *y for the residual update.
dlm_status mlp_sub_block(Runner& r, int l, int T, GemmOut* y) {
  dlm_ctx* ctx = r.ctx;
  const dlm_config& c = ctx->cfg;
  const int d = c.d, F = c.ffn;
  const long pad = split_pad(T);
  const dlm_layer_weights& W = ctx->layers[l];
  if (ctx->fp4) {  // input quantized by the residual+RMSNorm before
    TRY(r.gemm_fp4(A_PAIR, W.q_gate, &W.q_up, ctx->sf + l * (ctx->sf_pair + ctx->sf_down), T, F, d, y));
  } else {
    TRY(r.gemm_partial(A_PAIR, W.w_gate, W.w_up, ctx->xn, T, F, d, y));
  }
  EpiArgs es{};
  es.op = EPI_SILU;
  es.act = ctx->act;
  es.act_lo = pad * F;
  es.act_amax = ctx->fp4 ? ctx->act_amax : nullptr;
  TRY(finish_tiles(r, *y, F, es));
  if (ctx->fp4) {
    ActQuantArgs q{};
    q.xb = ctx->act;
    q.xb_lo = pad * F;
    q.K = F;
    q.codes = ctx->xcodes;
    q.scales = ctx->xscales;
    q.sx = ctx->sx;
    q.amax = ctx->act_amax;
    q.n_amax = (F + 63) / 64;
    q.T = T;
    CU_LAUNCH(launch_k(k_act_quant_wide, dim3((unsigned)((F / 16 + 255) / 256), T), dim3(256), 0, r.s, q));
    return r.gemm_fp4(A_KMAJOR, W.q_down, nullptr, ctx->sf + l * (ctx->sf_pair + ctx->sf_down) + ctx->sf_pair, T, d,
                      F, y);
  }
  return r.gemm_partial(A_KMAJOR, W.w_down, nullptr, ctx->act, T, d, F, y);
}

// One forward pass of T tokens (round, KV-fill or prefill chunk), all on stream r.s:
//   [s -> split bf16 -> W_a GEMM] ; h = E[x] (+ W_a s) ; RMSNorm
//   per layer: QKV GEMM ; RoPE + K/V cache ; attention ; O GEMM ; residual + RMSNorm ;
//              gate/up GEMM ; SiLU gate ; down GEMM ; residual + RMSNorm (next gain)
//   round only: LM head with row statistics and s = P E (fused), or logits GEMM ; row
//   statistics + P ; P E GEMM
// The projections leave per-slot partial sums; the kernel after each one finishes them.
// With f.T_pend > 0 the rows of a pending committed block come first (see FwdSpec).
dlm_status forward(Runner& r, const FwdSpec& f) {
  dlm_ctx* ctx = r.ctx;
  const dlm_config& c = ctx->cfg;
  const int Tp = f.T_pend, T = Tp + f.T;  // all rows of the pass
  const int d = c.d, Hq = c.n_q_heads, Hkv = c.n_kv_heads, hd = c.head_dim;
  const int ho = Hq * hd, nqkv = (Hq + 2 * Hkv) * hd;
  const long pad = split_pad(T);  // low halves of split activations start `pad` rows down
  const void* first_gain = c.n_layers > 0 ? ctx->layers[0].attn_norm : ctx->w.final_norm;
  const int32_t* tok0 = Tp ? f.pend_tokens : f.tokens;  // token rows [0, Tp) then [Tp, T)
  const int32_t* tok1 = Tp ? f.tokens : nullptr;
  const int pos0 = f.pos0 - Tp;  // position of row 0 (eager); graph mode: *d_L - Tp
  GemmOut y;

  // embedding + residual adapter (the pending rows carry no residual: s = 0 there)
  if (f.s) {
    const long n = (long)f.T * d, zn = (long)Tp * d;
    CU_LAUNCH(launch_k(k_to_bf16, dim3((unsigned)((zn + n + 255) / 256)), dim3(256), 0, r.s, f.s, ctx->sbf, n,
                       pad * d, zn));
    TRY(r.gemm_partial(A_KMAJOR, ctx->w.w_adapter, nullptr, ctx->sbf, T, d, d, &y));
    TRY(resid_norm(r, T, &y, tok0, first_gain, false, tok1, Tp));
  } else {
    TRY(resid_norm(r, T, nullptr, tok0, first_gain, false, tok1, Tp));
  }

  // KV cache planes of layer l: [K|V][Hkv][max_ctx][hd] values (bf16, or e4m3 bytes followed,
  // after all layers' values, by the fp32 row scales [layer][K|V][Hkv][max_ctx])
  const bool kv8 = c.kv_fmt == DLM_KV_FP8;
  const size_t plane_rows = (size_t)Hkv * c.max_ctx;
  const size_t plane_bytes = plane_rows * hd * (kv8 ? 1 : 2);
  float* const kv_scales = kv8 ? reinterpret_cast<float*>(ctx->kv + (size_t)2 * c.n_layers * plane_bytes) : nullptr;
  for (int l = 0; l < c.n_layers; ++l) {
    const dlm_layer_weights& W = ctx->layers[l];
    uint8_t* kp = ctx->kv + (size_t)(2 * l) * plane_bytes;
    uint8_t* vp = ctx->kv + (size_t)(2 * l + 1) * plane_bytes;
    __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(kp);
    __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(vp);
    float* ks = kv8 ? kv_scales + (size_t)(2 * l) * plane_rows : nullptr;
    float* vs = kv8 ? kv_scales + (size_t)(2 * l + 1) * plane_rows : nullptr;
    TRY(r.gemm_partial(A_KMAJOR, W.w_qkv, nullptr, ctx->xn, T, nqkv, d, &y));
    EpiArgs eq{};
    eq.op = EPI_QKV;
    eq.q = ctx->q;
    eq.kc = kv8 ? nullptr : kc;
    eq.vc = kv8 ? nullptr : vc;
    eq.kc8 = kv8 ? kp : nullptr;
    eq.vc8 = kv8 ? vp : nullptr;
    eq.ks = ks;
    eq.vs = vs;
    eq.Hq = Hq;
    eq.Hkv = Hkv;
    eq.hd = hd;
    eq.max_ctx = c.max_ctx;
    eq.pos0 = pos0;
    eq.pos0_dev = f.dev_L ? ctx->d_L : nullptr;
    eq.pos_off = -Tp;
    eq.rope_tab = ctx->rope_tab;
    TRY(finish_tiles(r, y, nqkv, eq));
    // the last layer's K/V do not depend on anything after its QKV projection
    if (!f.lm_head && l == c.n_layers - 1) break;

    AttnArgs aa{};
    aa.q = ctx->q;
    aa.kc = kc;
    aa.vc = vc;
    aa.ks = ks;
    aa.vs = vs;
    aa.o = ctx->o;
    aa.o_lo = pad * ho;
    aa.part_o = ctx->attn_part;
    aa.T = T;
    aa.Hq = Hq;
    aa.Hkv = Hkv;
    aa.hd = hd;
    aa.max_ctx = c.max_ctx;
    aa.pos0 = pos0;
    aa.pos0_dev = f.dev_L ? ctx->d_L : nullptr;
    aa.pos_off = -Tp;
    aa.causal = f.causal ? 1 : 0;
    aa.blk = Tp ? Tp : 0;  // pending block, then the new block; else one block
    aa.max_splits = (T <= c.block_size) ? ctx->attn_splits_B
                                        : (T <= 2 * c.block_size ? ctx->attn_splits_2B : ctx->attn_splits_T);
    aa.part_ml = ctx->attn_part + (size_t)aa.max_splits * T * Hq * hd;
    aa.err = ctx->d_err;
    cudaError_t e = attention_launch(aa, r.s);
    if (e != cudaSuccess) return fail(ctx, DLM_ECUDA, "attention: %s", cudaGetErrorString(e));

    TRY(r.gemm_partial(A_KMAJOR, W.w_o, nullptr, ctx->o, T, d, ho, &y));
    TRY(resid_norm(r, T, &y, nullptr, W.mlp_norm, ctx->fp4));

    TRY(mlp_sub_block(r, l, T, &y));
    const bool last = l + 1 == c.n_layers;
    TRY(resid_norm(r, T, &y, nullptr, last ? ctx->w.final_norm : ctx->layers[l + 1].attn_norm,
                   last && ctx->fp4 && f.lm_head));
  }
  if (!f.lm_head) return DLM_OK;
  const int Tl = f.T;  // LM head rows: the new block's

  // LM head: logits (finished inside the GEMM: its tiles are mostly single-slot), row
  // statistics, P = softmax (split bf16), s = P E
  if (ctx->lmf && ctx->fp4) {
    // one pass over the NVFP4 E: the rows of x were quantized by the last residual+RMSNorm;
    // the round's own rows start at Tp (a pending block's rows come first)
    if (c.n_layers == 0) TRY(act_quant(r, T, ctx->xn, pad * d, d));
    char msg[256];
    cudaError_t e = lmhead_fused_f4_launch(ctx->w.q_embed, ctx->sf + c.n_layers * (ctx->sf_pair + ctx->sf_down),
                                           ctx->xcodes, kMaxF4Tokens, Tp, ctx->xscales, ctx->sx, Tl, c.vocab, d,
                                           c.mask_id, f.stats, f.s_out, ctx->lmf, ctx->d_err, r.s, msg, sizeof(msg));
    if (e != cudaSuccess) return fail(ctx, DLM_ECUDA, "fused nvfp4 lm head: %s %s", cudaGetErrorString(e), msg);
    return DLM_OK;
  }
  if (ctx->lmf && !ctx->fp4 && Tl <= 32) {
    // one pass over E: logits, row statistics and s = P E on the rows [Tp, T) of the split x
    char msg[256];
    cudaError_t e = lmhead_fused_launch(ctx->xn, (int)(2 * pad), Tp, (int)(pad + Tp), ctx->w.embed, nullptr, Tl,
                                        c.vocab, d, c.mask_id, f.stats, f.s_out, ctx->lmf, ctx->d_err, r.s, msg,
                                        sizeof(msg));
    if (e != cudaSuccess) return fail(ctx, DLM_ECUDA, "fused lm head: %s %s", cudaGetErrorString(e), msg);
    return DLM_OK;
  }
  if (Tp) return fail(ctx, DLM_EUNSUPPORTED, "a pending block needs the fused LM head");
  EpiArgs el{};
  el.op = EPI_STORE;
  el.out = ctx->logits;
  el.ld = c.vocab;
  if (ctx->fp4) {  // input quantized by the last residual+RMSNorm
    if (c.n_layers == 0) TRY(act_quant(r, T, ctx->xn, pad * d, d));
    TRY(r.gemm_fp4(A_KMAJOR, ctx->w.q_embed, nullptr, ctx->sf + c.n_layers * (ctx->sf_pair + ctx->sf_down), T,
                   c.vocab, d, &y));
    TRY(finish_tiles(r, y, c.vocab, el));
  } else {
    TRY(r.gemm(A_KMAJOR, ctx->w.embed, nullptr, ctx->xn, T, c.vocab, d, el));
  }
  RowStatsArgs rs{};
  rs.logits = ctx->logits;
  rs.ld = c.vocab;
  rs.V = c.vocab;
  rs.mask_id = c.mask_id;
  rs.chunk = kRowChunk;
  rs.part = ctx->rs_part;
  rs.stats = f.stats;
  rs.P = ctx->P;
  rs.P_lo = pad * c.vocab;
  const int nch = (c.vocab + kRowChunk - 1) / kRowChunk;
  CU_LAUNCH(launch_k(k_rowstats_part, dim3(nch, T), dim3(256), 0, r.s, rs));
  CU_LAUNCH(launch_k(k_rowstats_final, dim3(nch, T), dim3(256), 0, r.s, rs));
  // NVFP4: s = P (q sigma) scaled by the tensor scale of E
  TRY(r.gemm_partial(A_MNMAJOR, ctx->fp4 ? ctx->e_deq : ctx->w.embed, nullptr, ctx->P, T, d, c.vocab, &y));
  EpiArgs ep{};
  ep.op = EPI_STORE;
  ep.out = f.s_out;
  ep.ld = d;
  ep.scale = ctx->fp4 ? ctx->w.q_embed.tensor_scale : 0.f;
  return finish_tiles(r, y, d, ep);
}

// Whether the context can carry a pending block in the next round: the pass then has 2B
// rows (split GEMM inputs up to 128 rows; NVFP4 GEMM inputs up to 64, so B = 32 and the
// round's own rows are the second group of 32) and must use the fused LM head.
bool fold_supported(const dlm_ctx* ctx) {
  const dlm_config& c = ctx->cfg;
  return ctx->lmf != nullptr && 2 * c.block_size <= (ctx->fp4 ? kMaxF4Tokens : kMaxSplitTokens) &&
         c.block_size <= 32 && (!ctx->fp4 || c.block_size == 32);
}

dlm_status launch_commit(Runner& r, const dlm_block_state& st, float tau, int mode, int k,
                         bool use_cond, cudaGraphConditionalHandle h) {
  dlm_ctx* ctx = r.ctx;
  const dlm_config& c = r.ctx->cfg;
  CommitArgs ca{};
  ca.maxprob = st.stats.maxprob;
  ca.argmax = st.stats.argmax;
  ca.tokens = st.tokens;
  ca.committed = st.committed;
  ca.s = st.s;
  ca.round = st.round;
  ca.status = st.status;
  ca.B = c.block_size;
  ca.d = c.d;
  ca.tau = tau;
  ca.mode = mode;
  ca.k = k;
  ca.use_cond = use_cond ? 1 : 0;
  ca.cond = h;
  CU_LAUNCH(launch_k(k_commit, dim3(1), dim3(kCommitThreads), 0, r.s, ca));
  return r.check();
}

dlm_status check_commit_args(dlm_ctx* ctx, float tau, int mode, int k) {
  if (mode != DLM_COMMIT_THRESHOLD && mode != DLM_COMMIT_TOPK)
    return fail(ctx, DLM_EINVAL, "commit mode %d", mode);
  if (mode == DLM_COMMIT_THRESHOLD && std::isnan(tau)) return fail(ctx, DLM_EINVAL, "tau is NaN");
  if (mode == DLM_COMMIT_TOPK && k < 1) return fail(ctx, DLM_EINVAL, "tpf_k < 1");
  return DLM_OK;
}

dlm_block_state internal_state(dlm_ctx* ctx) {
  dlm_block_state st{};
  st.tokens = ctx->b_tokens;
  st.committed = ctx->b_committed;
  st.s = ctx->b_s;
  st.round = ctx->b_round;
  st.status = ctx->b_status;
  st.stats = ctx->b_stats;
  return st;
}

dlm_status launch_block_init(Runner& r, const dlm_block_state& st) {
  dlm_ctx* ctx = r.ctx;
  const dlm_config& c = r.ctx->cfg;
  BlockInitArgs ba{st.tokens, st.committed, st.s, st.round, st.status, c.block_size, c.d, c.mask_id};
  CU_LAUNCH(launch_k(k_block_init, dim3(64), dim3(256), 0, r.s, ba));
  return r.check();
}

// One graph per (commit mode, tau / k, variant):
//   GV_EAGER: init -> WHILE { round } -> KV-fill forward -> finish
//   GV_FIRST: init -> WHILE { round } -> finish (the block's KV-fill is left pending)
//   GV_FOLD:  init -> first round carrying the pending block (its commit sets the loop
//             condition) -> WHILE { round } -> finish (this block's KV-fill left pending)
// finish copies tokens and rounds out and advances the device prefix length by B.
// Captures what `body` enqueues on the capture stream into graph g after the nodes `deps`
// (cudaStreamBeginCaptureToGraph), and returns the capture's leaf nodes in *leaves.
template <class Body>
dlm_status capture_into(dlm_ctx* ctx, cudaGraph_t g, const std::vector<cudaGraphNode_t>& deps, Body body,
                        std::vector<cudaGraphNode_t>* leaves) {
  cudaStream_t cs = ctx->cap_stream;
  CU(cudaStreamBeginCaptureToGraph(cs, g, deps.empty() ? nullptr : deps.data(), nullptr, deps.size(),
                                   cudaStreamCaptureModeThreadLocal));
  dlm_status st = body();
  if (st == DLM_OK && leaves) {
    cudaStreamCaptureStatus cst;
    const cudaGraphNode_t* d = nullptr;
    size_t nd = 0;
    cudaError_t e = cudaStreamGetCaptureInfo(cs, &cst, nullptr, nullptr, &d, &nd);
    if (e == cudaSuccess) leaves->assign(d, d + nd);
    else st = fail(ctx, DLM_ECUDA, "capture info: %s", cudaGetErrorString(e));
  }
  cudaGraph_t same = nullptr;
  cudaError_t e = cudaStreamEndCapture(cs, &same);
  if (st != DLM_OK) return st;
  CU(e);
  return DLM_OK;
}

dlm_status build_block_graph(dlm_ctx* ctx, int mode, float tau, int k, int variant, GraphEntry* out) {
  cudaGraph_t g = nullptr;
  CU(cudaGraphCreate(&g, 0));
  cudaGraphConditionalHandle h;
  CU(cudaGraphConditionalHandleCreate(&h, g, 1, cudaGraphCondAssignDefault));
  Runner r{ctx, ctx->cap_stream, {}};
  dlm_block_state st = internal_state(ctx);
  const dlm_config& c = ctx->cfg;
  std::vector<cudaGraphNode_t> leaves;

  FwdSpec f{};
  f.T = c.block_size;
  f.tokens = st.tokens;
  f.s = st.s;
  f.dev_L = true;
  f.lm_head = true;
  f.stats = st.stats;
  f.s_out = st.s;
  // init [-> the first round carrying the pending block's rows; its commit sets the loop
  // condition]
  TRY(capture_into(ctx, g, {}, [&]() -> dlm_status {
    TRY(launch_block_init(r, st));
    if (variant != GV_FOLD) return DLM_OK;
    FwdSpec f1 = f;
    f1.T_pend = c.block_size;
    f1.pend_tokens = ctx->pend_tokens;
    TRY(forward(r, f1));
    return launch_commit(r, st, tau, mode, k, true, h);
  }, &leaves));

  // while node with one round as its body
  cudaGraphNode_t n_while;
  cudaGraphNodeParams cp = {};
  cp.type = cudaGraphNodeTypeConditional;
  cp.conditional.handle = h;
  cp.conditional.type = cudaGraphCondTypeWhile;
  cp.conditional.size = 1;
  CU(cudaGraphAddNode(&n_while, g, leaves.data(), leaves.size(), &cp));
  cudaGraph_t body = cp.conditional.phGraph_out[0];
  TRY(capture_into(ctx, body, {}, [&]() -> dlm_status {
    TRY(forward(r, f));
    return launch_commit(r, st, tau, mode, k, true, h);
  }, nullptr));

  // [KV-fill of the committed block,] the block outputs and L += B
  TRY(capture_into(ctx, g, {n_while}, [&]() -> dlm_status {
    if (variant == GV_EAGER) {
      FwdSpec kf{};
      kf.T = c.block_size;
      kf.tokens = st.tokens;
      kf.dev_L = true;
      TRY(forward(r, kf));
    }
    BlockFinishArgs fa{st.tokens, st.round, st.status, ctx->d_err, ctx->out_tokens, ctx->out_rounds,
                       ctx->d_L, variant == GV_EAGER ? nullptr : ctx->pend_tokens, c.block_size};
    CU_LAUNCH(launch_k(k_block_finish, dim3(1), dim3(64), 0, ctx->cap_stream, fa));
    return r.check();
  }, nullptr));
  cudaGraphExec_t ex;
  CU(cudaGraphInstantiate(&ex, g, 0));
  *out = GraphEntry{mode, tau, k, variant, g, ex};
  return DLM_OK;
}

// Sets the prefix length on the host and the device (no pending-fill handling).
dlm_status set_L(dlm_ctx* ctx, int L, cudaStream_t s) {
  CU_LAUNCH(launch_k(k_set_int, dim3(1), dim3(1), 0, s, ctx->d_L, L));
  CU(cudaGetLastError());
  ctx->L = L;
  return DLM_OK;
}

// Runs a pending KV-fill on its own: the clean forward of the pending block at positions
// [L - B, L) (no LM head).
dlm_status flush_pending(dlm_ctx* ctx, cudaStream_t s) {
  if (!ctx->pending) return DLM_OK;
  Runner r{ctx, s, {}};
  FwdSpec f{};
  f.T = ctx->cfg.block_size;
  f.tokens = ctx->pend_tokens;
  f.pos0 = ctx->L - ctx->cfg.block_size;
  TRY(forward(r, f));
  ctx->pending = false;
  return DLM_OK;
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

const char* dlm_version(void) { return "dlm-b200 0.1 (sm_100a)"; }

void dlm_debug_set_pdl(int on) { g_pdl = on != 0; }

size_t dlm_workspace_size(const dlm_config* cfg) {
  char msg[128];
  if (!valid_cfg(cfg, msg, sizeof(msg))) return 0;
  return carve(nullptr, *cfg, nullptr);
}

size_t dlm_kv_cache_size(const dlm_config* c) {
  char msg[128];
  if (!valid_cfg(c, msg, sizeof(msg))) return 0;
  const size_t rows = (size_t)2 * c->n_layers * c->n_kv_heads * c->max_ctx;
  return c->kv_fmt == DLM_KV_FP8 ? rows * c->head_dim + rows * 4 : rows * c->head_dim * 2;
}

dlm_status dlm_ctx_create(const dlm_config* cfg, const dlm_weights* w, void* d_workspace,
                          size_t ws_bytes, void* d_kv_cache, size_t kv_bytes, dlm_ctx** out) {
  char msg[256];
  if (!out) return DLM_EINVAL;
  *out = nullptr;
  if (!valid_cfg(cfg, msg, sizeof(msg)) || !w || !d_workspace || (!d_kv_cache && cfg->n_layers > 0))
    return DLM_EINVAL;
  const bool fp4 = cfg->weight_fmt == DLM_WEIGHTS_NVFP4;
  auto q_ok = [](const dlm_nvfp4_matrix& m) { return m.codes && m.scales && std::isfinite(m.tensor_scale); };
  if ((!fp4 && !w->embed) || (fp4 && !q_ok(w->q_embed)) || !w->w_adapter || !w->final_norm ||
      (cfg->n_layers > 0 && !w->layers))
    return DLM_EINVAL;
  for (int l = 0; l < cfg->n_layers; ++l) {
    const dlm_layer_weights& L = w->layers[l];
    if (!L.attn_norm || !L.w_qkv || !L.w_o || !L.mlp_norm) return DLM_EINVAL;
    if (!fp4 && (!L.w_gate || !L.w_up || !L.w_down)) return DLM_EINVAL;
    if (fp4 && (!q_ok(L.q_gate) || !q_ok(L.q_up) || !q_ok(L.q_down))) return DLM_EINVAL;
  }
  // NVFP4 GEMMs stream 256 reduction elements per stage: d and ffn must be multiples of 256
  if (fp4 && (cfg->d % 256 || cfg->ffn % 256)) return DLM_EUNSUPPORTED;
  if ((uintptr_t)d_workspace % 256) return DLM_EINVAL;
  if (ws_bytes < dlm_workspace_size(cfg)) return DLM_ENOMEM_WS;
  if (kv_bytes < dlm_kv_cache_size(cfg)) return DLM_ENOMEM_WS;
  dlm_ctx* ctx = new (std::nothrow) dlm_ctx();
  if (!ctx) return DLM_EINVAL;
  ctx->cfg = *cfg;
  ctx->w = *w;
  ctx->layers.assign(w->layers, w->layers + cfg->n_layers);
  ctx->w.layers = ctx->layers.data();
  ctx->ws = (uint8_t*)d_workspace;
  ctx->ws_bytes = ws_bytes;
  ctx->kv = (uint8_t*)d_kv_cache;
  ctx->kv_bytes = kv_bytes;
  carve(ctx, *cfg, ctx->ws);
  cudaError_t e = cudaStreamCreateWithFlags(&ctx->cap_stream, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->ws, 0, ws_bytes, ctx->cap_stream);
  if (e == cudaSuccess) {
    const long nrt = (long)cfg->max_ctx * (cfg->head_dim / 2);
    k_rope_table<<<(unsigned)((nrt + 255) / 256), 256, 0, ctx->cap_stream>>>(ctx->rope_tab, cfg->max_ctx,
                                                                          cfg->head_dim, (double)cfg->rope_theta);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && fp4 && ctx->e_deq) {
    // E for the embedding rows and P E of the unfused LM head: q sigma in bf16 (exact); the
    // tensor scale is applied where they are used
    const long nb = (long)cfg->vocab * (cfg->d / 16);
    k_nvfp4_dequant_bf16<<<(unsigned)((nb + 255) / 256), 256, 0, ctx->cap_stream>>>(
        (const uint8_t*)w->q_embed.codes, (const uint8_t*)w->q_embed.scales, nb, ctx->e_deq);
    e = cudaGetLastError();
  }
  // the weights' e4m3 scales, re-tiled for the FP4 MMA (tensor-memory scale layout)
  for (int l = 0; l < cfg->n_layers && fp4 && e == cudaSuccess; ++l) {
    uint8_t* base = ctx->sf + l * (ctx->sf_pair + ctx->sf_down);
    e = nvf4_sf_tile(w->layers[l].q_gate, &w->layers[l].q_up, cfg->ffn, cfg->d, A_PAIR, base, ctx->cap_stream);
    if (e == cudaSuccess)
      e = nvf4_sf_tile(w->layers[l].q_down, nullptr, cfg->d, cfg->ffn, A_KMAJOR, base + ctx->sf_pair, ctx->cap_stream);
  }
  if (e == cudaSuccess && fp4)
    e = nvf4_sf_tile(w->q_embed, nullptr, cfg->vocab, cfg->d, A_KMAJOR,
                     ctx->sf + cfg->n_layers * (ctx->sf_pair + ctx->sf_down), ctx->cap_stream);
  if (e == cudaSuccess) e = (cudaError_t)gemm_init_attributes();
  if (e == cudaSuccess && fp4) e = (cudaError_t)gemm_fp4_init_attributes();
  if (e == cudaSuccess) e = (cudaError_t)attention_init_attributes();
  if (e == cudaSuccess) e = (cudaError_t)ops_init_attributes();
  if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->cap_stream);
  if (e != cudaSuccess) {
    if (ctx->cap_stream) cudaStreamDestroy(ctx->cap_stream);
    delete ctx;
    return DLM_ECUDA;
  }
  *out = ctx;
  return DLM_OK;
}

dlm_status dlm_ctx_destroy(dlm_ctx* ctx) {
  if (!ctx) return DLM_EINVAL;
  for (auto& g : ctx->graphs) {
    cudaGraphExecDestroy(g.exec);
    cudaGraphDestroy(g.graph);
  }
  if (ctx->cap_stream) cudaStreamDestroy(ctx->cap_stream);
  delete ctx;
  return DLM_OK;
}

const char* dlm_last_error(const dlm_ctx* ctx) { return ctx ? ctx->err.c_str() : "null context"; }

int dlm_prefix_len(const dlm_ctx* ctx) { return ctx ? ctx->L : -1; }

dlm_status dlm_set_prefix_len(dlm_ctx* ctx, int L, void* stream) {
  if (!ctx) return DLM_EINVAL;
  if (L < 0 || L > ctx->cfg.max_ctx) return fail(ctx, DLM_EINVAL, "L=%d", L);
  if (ctx->pending) {
    // the pending block's rows [L_old - B, L_old): free when the new prefix ends before them,
    // else written now
    if (L <= ctx->L - ctx->cfg.block_size) ctx->pending = false;
    else TRY(flush_pending(ctx, (cudaStream_t)stream));
  }
  return set_L(ctx, L, (cudaStream_t)stream);
}

dlm_status dlm_kv_flush(dlm_ctx* ctx, void* stream) {
  if (!ctx) return DLM_EINVAL;
  return flush_pending(ctx, (cudaStream_t)stream);
}

dlm_status dlm_set_fill_mode(dlm_ctx* ctx, int mode, void* stream) {
  if (!ctx) return DLM_EINVAL;
  if (mode != DLM_FILL_EAGER && mode != DLM_FILL_DEFERRED) return fail(ctx, DLM_EINVAL, "fill mode %d", mode);
  if (mode == DLM_FILL_EAGER) TRY(flush_pending(ctx, (cudaStream_t)stream));
  ctx->fill_deferred = mode == DLM_FILL_DEFERRED;
  return DLM_OK;
}

int dlm_fill_pending(const dlm_ctx* ctx) { return ctx ? (ctx->pending ? 1 : 0) : -1; }

dlm_status dlm_prefill(dlm_ctx* ctx, const int32_t* d_tokens, int n, void* stream) {
  if (!ctx) return DLM_EINVAL;
  if (!d_tokens || n < 0) return fail(ctx, DLM_EINVAL, "prefill args");
  if (ctx->L + n > ctx->cfg.max_ctx) return fail(ctx, DLM_EKVCAP, "prefill: %d + %d > %d", ctx->L, n, ctx->cfg.max_ctx);
  TRY(flush_pending(ctx, (cudaStream_t)stream));
  Runner r{ctx, (cudaStream_t)stream, {}};
  const int chunk = prefill_chunk(ctx->cfg);
  for (int off = 0; off < n; off += chunk) {
    int T = n - off < chunk ? n - off : chunk;
    FwdSpec f{};
    f.T = T;
    f.tokens = d_tokens + off;
    f.pos0 = ctx->L + off;
    f.causal = true;
    TRY(forward(r, f));
  }
  return set_L(ctx, ctx->L + n, (cudaStream_t)stream);
}

dlm_status dlm_block_init(dlm_ctx* ctx, const dlm_block_state* st, void* stream) {
  if (!ctx) return DLM_EINVAL;
  if (!st || !st->tokens || !st->committed || !st->s || !st->round) return fail(ctx, DLM_EINVAL, "block state");
  Runner r{ctx, (cudaStream_t)stream, {}};
  return launch_block_init(r, *st);
}

dlm_status dlm_round(dlm_ctx* ctx, const dlm_block_state* st, float tau, int commit_mode, int tpf_k,
                     void* stream) {
  if (!ctx) return DLM_EINVAL;
  if (!st || !st->tokens || !st->committed || !st->s || !st->round || !st->stats.m || !st->stats.lse ||
      !st->stats.maxprob || !st->stats.entropy || !st->stats.argmax)
    return fail(ctx, DLM_EINVAL, "block state");
  TRY(check_commit_args(ctx, tau, commit_mode, tpf_k));
  const dlm_config& c = ctx->cfg;
  if (ctx->L + c.block_size > c.max_ctx)
    return fail(ctx, DLM_EKVCAP, "round: L %d + B %d > %d", ctx->L, c.block_size, c.max_ctx);
  Runner r{ctx, (cudaStream_t)stream, {}};
  FwdSpec f{};
  f.T = c.block_size;
  f.tokens = st->tokens;
  f.s = st->s;
  f.pos0 = ctx->L;
  f.lm_head = true;
  f.stats = st->stats;
  f.s_out = st->s;
  if (ctx->pending) {  // the pending KV-fill rides along (see FwdSpec)
    f.T_pend = c.block_size;
    f.pend_tokens = ctx->pend_tokens;
  }
  TRY(forward(r, f));
  ctx->pending = false;
  return launch_commit(r, *st, tau, commit_mode, tpf_k, false, 0);
}

dlm_status dlm_kv_fill(dlm_ctx* ctx, const int32_t* d_tokens, void* stream) {
  if (!ctx) return DLM_EINVAL;
  if (!d_tokens) return fail(ctx, DLM_EINVAL, "kv_fill tokens");
  const dlm_config& c = ctx->cfg;
  if (ctx->L + c.block_size > c.max_ctx) return fail(ctx, DLM_EKVCAP, "kv_fill: capacity");
  cudaStream_t s = (cudaStream_t)stream;
  TRY(flush_pending(ctx, s));  // at most one block pending
  if (ctx->fill_deferred && fold_supported(ctx)) {
    // deferred: keep the tokens; the next round (or dlm_kv_flush) writes the rows
    CU(cudaMemcpyAsync(ctx->pend_tokens, d_tokens, (size_t)c.block_size * 4, cudaMemcpyDeviceToDevice, s));
    TRY(set_L(ctx, ctx->L + c.block_size, s));
    ctx->pending = true;
    return DLM_OK;
  }
  Runner r{ctx, s, {}};
  FwdSpec f{};
  f.T = c.block_size;
  f.tokens = d_tokens;
  f.pos0 = ctx->L;
  TRY(forward(r, f));
  return set_L(ctx, ctx->L + c.block_size, s);
}

dlm_status dlm_mlp_block(dlm_ctx* ctx, int layer, const float* d_h_in, float* d_h_out, int T, void* stream) {
  if (!ctx) return DLM_EINVAL;
  const dlm_config& c = ctx->cfg;
  const int tmax = ctx->fp4 ? kMaxF4Tokens : ctx->Tmax;
  if (!d_h_in || !d_h_out || layer < 0 || layer >= c.n_layers || T < 1 || T > tmax)
    return fail(ctx, DLM_EINVAL, "mlp_block: layer %d, T %d", layer, T);
  cudaStream_t s = (cudaStream_t)stream;
  Runner r{ctx, s, {}};
  const size_t bytes = (size_t)T * c.d * sizeof(float);
  CU(cudaMemcpyAsync(ctx->h, d_h_in, bytes, cudaMemcpyDeviceToDevice, s));
  // h unchanged (no projection to add), xn = RMSNorm(h) g_mlp (quantized for NVFP4 weights)
  TRY(resid_norm(r, T, nullptr, nullptr, ctx->layers[layer].mlp_norm, ctx->fp4));
  GemmOut y;
  TRY(mlp_sub_block(r, layer, T, &y));
  const bool last = layer + 1 == c.n_layers;
  TRY(resid_norm(r, T, &y, nullptr, last ? ctx->w.final_norm : ctx->layers[layer + 1].attn_norm));
  CU(cudaMemcpyAsync(d_h_out, ctx->h, bytes, cudaMemcpyDeviceToDevice, s));
  return DLM_OK;
}

dlm_status dlm_decode_block(dlm_ctx* ctx, float tau, int commit_mode, int tpf_k, int32_t* d_tokens_out,
                            int32_t* d_rounds_out, void* stream) {
  if (!ctx) return DLM_EINVAL;
  TRY(check_commit_args(ctx, tau, commit_mode, tpf_k));
  const dlm_config& c = ctx->cfg;
  if (ctx->L + c.block_size > c.max_ctx)
    return fail(ctx, DLM_EKVCAP, "decode_block: L %d + B %d > %d", ctx->L, c.block_size, c.max_ctx);
  cudaStream_t s = (cudaStream_t)stream;
  const bool defer = ctx->fill_deferred && fold_supported(ctx);
  if (!defer) TRY(flush_pending(ctx, s));
  const int variant = !defer ? GV_EAGER : (ctx->pending ? GV_FOLD : GV_FIRST);
  GraphEntry* ge = nullptr;
  for (auto& g : ctx->graphs)
    if (g.mode == commit_mode && g.variant == variant && (commit_mode == DLM_COMMIT_TOPK ? g.k == tpf_k : g.tau == tau))
      ge = &g;
  if (!ge) {
    GraphEntry ne{};
    TRY(build_block_graph(ctx, commit_mode, tau, tpf_k, variant, &ne));
    ctx->graphs.push_back(ne);
    ge = &ctx->graphs.back();
  }
  CU(cudaGraphLaunch(ge->exec, s));
  if (d_tokens_out) CU(cudaMemcpyAsync(d_tokens_out, ctx->out_tokens, c.block_size * 4, cudaMemcpyDeviceToDevice, s));
  if (d_rounds_out) CU(cudaMemcpyAsync(d_rounds_out, ctx->out_rounds, 2 * 4, cudaMemcpyDeviceToDevice, s));
  ctx->L += c.block_size;
  ctx->pending = defer;
  return DLM_OK;
}

dlm_status dlm_generate(dlm_ctx* ctx, const int32_t* h_prompt, int prompt_len, int max_new, float tau,
                        int commit_mode, int tpf_k, int32_t* h_tokens_out, int32_t* h_rounds_per_block,
                        dlm_timing* h_timing, void* stream) {
  if (!ctx) return DLM_EINVAL;
  if ((!h_prompt && prompt_len > 0) || prompt_len < 0 || max_new < 0 || (!h_tokens_out && max_new > 0))
    return fail(ctx, DLM_EINVAL, "generate args");
  TRY(check_commit_args(ctx, tau, commit_mode, tpf_k));
  const dlm_config& c = ctx->cfg;
  const int B = c.block_size;
  const int nblk = (max_new + B - 1) / B;
  if ((long)prompt_len + (long)nblk * B > c.max_ctx)
    return fail(ctx, DLM_EKVCAP, "generate: %d + %d blocks of %d > %d", prompt_len, nblk, B, c.max_ctx);
  cudaStream_t s = (cudaStream_t)stream;
  auto t0 = std::chrono::steady_clock::now();
  TRY(dlm_set_prefix_len(ctx, 0, stream));
  if (prompt_len > 0) {
    CU(cudaMemcpyAsync(ctx->tok_buf, h_prompt, (size_t)prompt_len * 4, cudaMemcpyHostToDevice, s));
    TRY(dlm_prefill(ctx, ctx->tok_buf, prompt_len, stream));
  }
  CU(cudaStreamSynchronize(s));
  auto t1 = std::chrono::steady_clock::now();
  int total_rounds = 0;
  int32_t rb[2];
  for (int b = 0; b < nblk; ++b) {
    TRY(dlm_decode_block(ctx, tau, commit_mode, tpf_k, nullptr, nullptr, stream));
    const int keep = (max_new - b * B) < B ? (max_new - b * B) : B;
    CU(cudaMemcpyAsync(h_tokens_out + (size_t)b * B, ctx->out_tokens, (size_t)keep * 4, cudaMemcpyDeviceToHost, s));
    CU(cudaMemcpyAsync(rb, ctx->out_rounds, 8, cudaMemcpyDeviceToHost, s));
    CU(cudaStreamSynchronize(s));
    if (rb[1] != 0) return fail(ctx, rb[1], "block %d: device status %d", b, rb[1]);
    if (h_rounds_per_block) h_rounds_per_block[b] = rb[0];
    total_rounds += rb[0];
  }
  TRY(flush_pending(ctx, s));  // the last block's KV-fill: the cache is complete on return
  CU(cudaStreamSynchronize(s));
  auto t2 = std::chrono::steady_clock::now();
  if (h_timing) {
    h_timing->prefill_ms = std::chrono::duration<double, std::milli>(t1 - t0).count();
    h_timing->decode_ms = std::chrono::duration<double, std::milli>(t2 - t1).count();
    h_timing->n_blocks = nblk;
    h_timing->n_rounds = total_rounds;
  }
  return DLM_OK;
}

// ------------------------------------------------------------------ single operations
}  // extern "C"

// ------------------------------------------------------------------ single operations
// Scratch of a single-operation call: [256 B status][tile counters][GEMM partials][extras].
static size_t op_header() { return 256; }
static size_t op_counters(int N) { return align256((size_t)((N + 63) / 64 + 2) * 4); }

struct OpScratch {
  uint8_t* base;
  size_t off;
  int* err;
  int* cnt;
  float* partial;
  OpScratch(void* p, int n_cnt, size_t partial_bytes) : base((uint8_t*)p) {
    err = (int*)base;
    cnt = (int*)(base + op_header());
    partial = (float*)(base + op_header() + op_counters(n_cnt));
    off = op_header() + op_counters(n_cnt) + align256(partial_bytes);
  }
  template <class T>
  T* take(size_t count) {
    T* q = (T*)(base + off);
    off += align256(count * sizeof(T));
    return q;
  }
};

static dlm_status op_gemm(const GemmPlan& plan0, EpiArgs epi, const OpScratch& sc, cudaStream_t s) {
  dlm_ctx* ctx = nullptr;
  GemmPlan p = plan0;
  epi.tile_cnt = sc.cnt;
  p.epi = epi;
  CU(gemm_launch(p, sc.err, s));
  return DLM_OK;
}

static size_t lmhead_partial(int B, int V, int d) {
  size_t lm = gemm_partial_bytes(B, V, d, A_KMAJOR), pe = gemm_partial_bytes(B, d, V, A_MNMAJOR);
  return lm > pe ? lm : pe;
}

extern "C" {

size_t dlm_gemm_scratch_size(int T, int N, int K) {
  return op_header() + op_counters(N) + align256(gemm_partial_bytes(T, N, K, A_KMAJOR));
}

static dlm_status gemm_op(const void* d_x, const void* d_w, float* d_y, int T, int N, int K, void* d_scratch,
                          size_t scratch_bytes, void* stream, bool split) {
  dlm_ctx* ctx = nullptr;
  if (!d_x || !d_w || !d_scratch || T < 1 || T > (split ? kMaxSplitTokens : kMaxTokens) || N < 1 || K < 64 ||
      K % 8)
    return DLM_EINVAL;
  if (scratch_bytes < dlm_gemm_scratch_size(T, N, K)) return DLM_ENOMEM_WS;
  CU((cudaError_t)gemm_init_attributes());
  cudaStream_t s = (cudaStream_t)stream;
  OpScratch sc(d_scratch, N, gemm_partial_bytes(T, N, K, A_KMAJOR));
  char msg[256];
  GemmPlan p;
  if (!gemm_plan(&p, A_KMAJOR, d_w, nullptr, d_x, T, N, K, sc.partial, msg, sizeof(msg), split))
    return DLM_EUNSUPPORTED;
  // the status word and tile counters start at zero (a partial-sums-only call uses neither)
  if (d_y) CU(cudaMemsetAsync(d_scratch, 0, op_header() + op_counters(N), s));
  EpiArgs e{};
  e.op = d_y ? EPI_STORE : EPI_PARTIAL;  // no output: the tensor-core kernel alone
  e.out = d_y;
  e.ld = N;
  return op_gemm(p, e, sc, s);
}

dlm_status dlm_gemm_bf16(const void* d_x, const void* d_w, float* d_y, int T, int N, int K, void* d_scratch,
                         size_t scratch_bytes, void* stream) {
  return gemm_op(d_x, d_w, d_y, T, N, K, d_scratch, scratch_bytes, stream, false);
}

int dlm_split_pad(int T) { return split_pad(T); }

dlm_status dlm_gemm_bf16x2(const void* d_x2, const void* d_w, float* d_y, int T, int N, int K, void* d_scratch,
                           size_t scratch_bytes, void* stream) {
  return gemm_op(d_x2, d_w, d_y, T, N, K, d_scratch, scratch_bytes, stream, true);
}

size_t dlm_gemm_f32_scratch_size(int T, int N, int K) {
  if (T < 1 || T > kMaxSplitTokens || K < 1) return 0;
  return dlm_gemm_scratch_size(T, N, K) + align256((size_t)2 * split_pad(T) * K * 2);
}

dlm_status dlm_gemm_f32(const float* d_x, const void* d_w, float* d_y, int T, int N, int K, void* d_scratch,
                        size_t scratch_bytes, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_x || !d_w || !d_y || !d_scratch || T < 1 || T > kMaxSplitTokens || N < 1 || K < 64 || K % 8)
    return DLM_EINVAL;
  if (scratch_bytes < dlm_gemm_f32_scratch_size(T, N, K)) return DLM_ENOMEM_WS;
  cudaStream_t s = (cudaStream_t)stream;
  // the split pair x = hi + lo goes after the GEMM's own scratch: rows [0, T) high halves,
  // rows [pad, pad + T) low halves, the padding rows zero
  const size_t gemm_sc = dlm_gemm_scratch_size(T, N, K);
  const long pad = split_pad(T);
  __nv_bfloat16* x2 = (__nv_bfloat16*)((uint8_t*)d_scratch + gemm_sc);
  CU(cudaMemsetAsync(x2, 0, (size_t)2 * pad * K * 2, s));
  const long n = (long)T * K;
  CU_LAUNCH(launch_k(k_to_bf16, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, d_x, x2, n, pad * K, 0L));
  return gemm_op(x2, d_w, d_y, T, N, K, d_scratch, gemm_sc, stream, true);
}

size_t dlm_lmhead_scratch_size(int B, int V, int d) {
  const int nch = (V + kRowChunk - 1) / kRowChunk;
  size_t unfused = op_header() + op_counters(V > d ? V : d) + align256(lmhead_partial(B, V, d)) +
                   align256((size_t)B * V * 4) + align256((size_t)2 * split_pad(B) * V * 2) +
                   align256((size_t)16 * B * nch);
  if (!lmhead_fused_supported(B, d)) return unfused;
  size_t fused = op_header() + align256((size_t)64 * d * 2) + align256(lmhead_fused_scratch_bytes(V, d));
  return fused > unfused ? fused : unfused;
}

dlm_status dlm_lmhead_rowstats(const void* d_x, const void* d_embed, int B, int V, int d, int mask_id,
                               const void* d_p_given, dlm_row_stats stats, float* d_s, void* d_scratch,
                               size_t scratch_bytes, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_x || !d_embed || !d_s || !d_scratch || B < 1 || B > kMaxSplitTokens || V < 2 || V % 8 || d < 64 ||
      d % 64 || !stats.m || !stats.lse || !stats.maxprob || !stats.entropy || !stats.argmax)
    return DLM_EINVAL;
  if (scratch_bytes < dlm_lmhead_scratch_size(B, V, d)) return DLM_ENOMEM_WS;
  cudaStream_t s = (cudaStream_t)stream;
  if (lmhead_fused_supported(B, d)) {
    // one pass over E; x as the split pair the kernel reads (high halves = x, low halves 0)
    uint8_t* base = (uint8_t*)d_scratch;
    void* x2 = base + op_header();
    void* lmf = base + op_header() + align256((size_t)64 * d * 2);
    CU(cudaMemsetAsync(base, 0, op_header() + (size_t)64 * d * 2, s));
    CU(cudaMemcpyAsync(x2, d_x, (size_t)B * d * 2, cudaMemcpyDeviceToDevice, s));
    char msg[256];
    cudaError_t e = lmhead_fused_launch(x2, 64, 0, 32, d_embed, d_p_given, B, V, d, mask_id, stats, d_s, lmf,
                                        (int*)base, s, msg, sizeof(msg));
    return e == cudaSuccess ? DLM_OK : DLM_ECUDA;
  }
  CU((cudaError_t)gemm_init_attributes());
  const int nch = (V + kRowChunk - 1) / kRowChunk;
  OpScratch sc(d_scratch, V > d ? V : d, lmhead_partial(B, V, d));
  float* logits = sc.take<float>((size_t)B * V);
  __nv_bfloat16* P = sc.take<__nv_bfloat16>((size_t)2 * split_pad(B) * V);
  float* part = sc.take<float>((size_t)4 * B * nch);
  CU(cudaMemsetAsync(d_scratch, 0, op_header() + op_counters(V > d ? V : d), s));
  char msg[256];
  GemmPlan p;
  if (!gemm_plan(&p, A_KMAJOR, d_embed, nullptr, d_x, B, V, d, sc.partial, msg, sizeof(msg))) return DLM_EUNSUPPORTED;
  EpiArgs el{};
  el.op = EPI_STORE;
  el.out = logits;
  el.ld = V;
  TRY(op_gemm(p, el, sc, s));
  RowStatsArgs rs{};
  rs.logits = logits;
  rs.ld = V;
  rs.V = V;
  rs.mask_id = mask_id;
  rs.chunk = kRowChunk;
  rs.part = part;
  rs.stats = stats;
  rs.P = d_p_given ? nullptr : P;
  rs.P_lo = (long)split_pad(B) * V;  // own softmax: split bf16 pair; a given P is plain bf16
  CU_LAUNCH(launch_k(k_rowstats_part, dim3(nch, B), dim3(256), 0, s, rs));
  CU_LAUNCH(launch_k(k_rowstats_final, dim3(nch, B), dim3(256), 0, s, rs));
  GemmPlan q;
  if (!gemm_plan(&q, A_MNMAJOR, d_embed, nullptr, d_p_given ? d_p_given : P, B, d, V, sc.partial, msg, sizeof(msg),
                 d_p_given == nullptr))
    return DLM_EUNSUPPORTED;
  EpiArgs ep{};
  ep.op = EPI_STORE;
  ep.out = d_s;
  ep.ld = d;
  return op_gemm(q, ep, sc, s);
}

size_t dlm_adapter_scratch_size(int B, int d) {
  return op_header() + op_counters(d) + align256(gemm_partial_bytes(B, d, d, A_KMAJOR)) +
         align256((size_t)2 * split_pad(B) * d * 2) + align256((size_t)((d + 127) / 128) * B * 4);
}

dlm_status dlm_adapter_embed(const void* d_embed, const void* d_w_adapter, const int32_t* d_tokens,
                             const float* d_s, float* d_h0, int B, int d, void* d_scratch, size_t scratch_bytes,
                             void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_embed || !d_w_adapter || !d_tokens || !d_s || !d_h0 || !d_scratch || B < 1 || B > kMaxSplitTokens ||
      d < 64 || d % 64)
    return DLM_EINVAL;
  if (scratch_bytes < dlm_adapter_scratch_size(B, d)) return DLM_ENOMEM_WS;
  CU((cudaError_t)gemm_init_attributes());
  cudaStream_t s = (cudaStream_t)stream;
  OpScratch sc(d_scratch, d, gemm_partial_bytes(B, d, d, A_KMAJOR));
  __nv_bfloat16* sbf = sc.take<__nv_bfloat16>((size_t)2 * split_pad(B) * d);
  float* ss = sc.take<float>((size_t)((d + 127) / 128) * B);
  CU(cudaMemsetAsync(d_scratch, 0, op_header() + op_counters(d), s));
  long n = (long)B * d;
  CU_LAUNCH(launch_k(k_to_bf16, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, d_s, sbf, n,
                     (long)split_pad(B) * d, 0L));
  char msg[256];
  GemmPlan p;
  if (!gemm_plan(&p, A_KMAJOR, d_w_adapter, nullptr, sbf, B, d, d, sc.partial, msg, sizeof(msg), true))
    return DLM_EUNSUPPORTED;
  EpiArgs e{};
  e.op = EPI_EMBED;
  e.h = d_h0;
  e.ss = ss;
  e.embed = (const __nv_bfloat16*)d_embed;
  e.tokens = d_tokens;
  return op_gemm(p, e, sc, s);
}

size_t dlm_attention_scratch_size(int T, int Hq, int hd, int max_ctx) {
  int sp = attention_split_cap(T, max_ctx);  // upper bound of the split count
  return op_header() + align256(attention_scratch_bytes(T, Hq, hd, sp));
}

dlm_status dlm_bd_attention(const void* d_q, const void* d_k_cache, const void* d_v_cache, void* d_o, int T,
                            int L, int Hq, int Hkv, int hd, int max_ctx, int causal, void* d_scratch,
                            size_t scratch_bytes, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_q || !d_k_cache || !d_v_cache || !d_o || !d_scratch || T < 1 || L < 0 || Hq < 1 || Hkv < 1 ||
      Hq % Hkv || !(hd == 32 || hd == 64 || hd == 128) || L + T > max_ctx)
    return DLM_EINVAL;
  if (scratch_bytes < dlm_attention_scratch_size(T, Hq, hd, max_ctx)) return DLM_ENOMEM_WS;
  CU((cudaError_t)attention_init_attributes());
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* sc = (uint8_t*)d_scratch;
  AttnArgs a{};
  a.q = (const __nv_bfloat16*)d_q;
  a.kc = (const __nv_bfloat16*)d_k_cache;
  a.vc = (const __nv_bfloat16*)d_v_cache;
  a.o = (__nv_bfloat16*)d_o;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.hd = hd;
  a.max_ctx = max_ctx;
  a.pos0 = L;
  a.causal = causal ? 1 : 0;
  a.max_splits = attention_max_splits(T, Hq, Hkv, max_ctx);
  a.part_o = (float*)(sc + op_header());
  a.part_ml = a.part_o + (size_t)a.max_splits * T * Hq * hd;
  a.err = nullptr;  // the attention kernels have no waits and report nothing on the device
  CU(attention_launch(a, s));
  return DLM_OK;
}

dlm_status dlm_bd_attention_fp8(const void* d_q, const void* d_k_codes, const float* d_k_scales, const void* d_v_codes,
                                const float* d_v_scales, void* d_o, int T, int L, int Hq, int Hkv, int hd, int max_ctx,
                                int causal, void* d_scratch, size_t scratch_bytes, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_q || !d_k_codes || !d_v_codes || !d_k_scales || !d_v_scales || !d_o || !d_scratch || T < 1 || L < 0 ||
      Hq < 1 || Hkv < 1 || Hq % Hkv || !(hd == 32 || hd == 64 || hd == 128) || L + T > max_ctx || max_ctx % 4)
    return DLM_EINVAL;
  if (scratch_bytes < dlm_attention_scratch_size(T, Hq, hd, max_ctx)) return DLM_ENOMEM_WS;
  CU((cudaError_t)attention_init_attributes());
  uint8_t* sc = (uint8_t*)d_scratch;
  AttnArgs a{};
  a.q = (const __nv_bfloat16*)d_q;
  a.kc = (const __nv_bfloat16*)d_k_codes;
  a.vc = (const __nv_bfloat16*)d_v_codes;
  a.ks = d_k_scales;
  a.vs = d_v_scales;
  a.o = (__nv_bfloat16*)d_o;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.hd = hd;
  a.max_ctx = max_ctx;
  a.pos0 = L;
  a.causal = causal ? 1 : 0;
  a.max_splits = attention_max_splits(T, Hq, Hkv, max_ctx);
  a.part_o = (float*)(sc + op_header());
  a.part_ml = a.part_o + (size_t)a.max_splits * T * Hq * hd;
  CU(attention_launch(a, (cudaStream_t)stream));
  return DLM_OK;
}

dlm_status dlm_commit(const float* d_maxprob, const int32_t* d_argmax, int32_t* d_tokens, uint8_t* d_committed,
                      float* d_s, int32_t* d_round, int32_t* d_status, int B, int d, float tau, int commit_mode,
                      int tpf_k, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_maxprob || !d_argmax || !d_tokens || !d_committed || !d_s || !d_round || B < 1 || B > 64 || d < 1)
    return DLM_EINVAL;
  if (commit_mode != DLM_COMMIT_THRESHOLD && commit_mode != DLM_COMMIT_TOPK) return DLM_EINVAL;
  if (commit_mode == DLM_COMMIT_THRESHOLD && std::isnan(tau)) return DLM_EINVAL;
  if (commit_mode == DLM_COMMIT_TOPK && tpf_k < 1) return DLM_EINVAL;
  CommitArgs ca{};
  ca.maxprob = d_maxprob;
  ca.argmax = d_argmax;
  ca.tokens = d_tokens;
  ca.committed = d_committed;
  ca.s = d_s;
  ca.round = d_round;
  ca.status = d_status;
  ca.B = B;
  ca.d = d;
  ca.tau = tau;
  ca.mode = commit_mode;
  ca.k = tpf_k;
  CU_LAUNCH(launch_k(k_commit, dim3(1), dim3(kCommitThreads), 0, (cudaStream_t)stream, ca));
  return cudaGetLastError() == cudaSuccess ? DLM_OK : DLM_ECUDA;
}

dlm_status dlm_nvfp4_quantize(const void* d_w, int rows, int cols, void* d_codes, void* d_scales,
                              float* d_tensor_scale, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_w || !d_codes || !d_scales || !d_tensor_scale || rows < 1 || cols < 16 || cols % 16) return DLM_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(d_tensor_scale, 0, 4, s) != cudaSuccess) return DLM_ECUDA;
  long n = (long)rows * cols;
  CU_LAUNCH(launch_k(k_amax_bf16, dim3(1024), dim3(256), 0, s, (const __nv_bfloat16*)d_w, n, (unsigned*)d_tensor_scale));
  long nblk = (long)rows * (cols / 16);
  CU_LAUNCH(launch_k(k_nvfp4_quantize, dim3((unsigned)((nblk + 255) / 256)), dim3(256), 0, s, (const __nv_bfloat16*)d_w, rows, cols,
                                                                  (uint8_t*)d_codes, (uint8_t*)d_scales,
                                                                  (const unsigned*)d_tensor_scale, nullptr));
  CU_LAUNCH(launch_k(k_amax_to_scale, dim3(1), dim3(1), 0, s, d_tensor_scale));
  return cudaGetLastError() == cudaSuccess ? DLM_OK : DLM_ECUDA;
}

size_t dlm_lmhead_nvfp4_scratch_size(int B, int V, int d) {
  if (!lmhead_fused_f4_supported(B, d) || V < 2) return 0;
  return op_header() + align256((size_t)kMaxF4Tokens * d / 2) + align256(f4_scale_bytes(d)) +
         align256(kMaxF4Tokens * 4) + align256(nvf4_sf_tile_bytes(V, d, A_KMAJOR)) +
         align256(lmhead_fused_scratch_bytes(V, d));
}

dlm_status dlm_lmhead_rowstats_nvfp4(const float* d_x, const dlm_nvfp4_matrix* E, int B, int V, int d, int mask_id,
                                     dlm_row_stats stats, float* d_s, void* d_scratch, size_t scratch_bytes,
                                     void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_x || !E || !E->codes || !E->scales || !std::isfinite(E->tensor_scale) || !d_s || !d_scratch || B < 1 ||
      V < 2 || d < 64 || !stats.m || !stats.lse || !stats.maxprob || !stats.entropy || !stats.argmax)
    return DLM_EINVAL;
  if (!lmhead_fused_f4_supported(B, d)) return DLM_EUNSUPPORTED;
  if (scratch_bytes < dlm_lmhead_nvfp4_scratch_size(B, V, d)) return DLM_ENOMEM_WS;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* base = (uint8_t*)d_scratch;
  size_t off = op_header();
  auto take = [&](size_t bytes) {
    uint8_t* q = base + off;
    off += align256(bytes);
    return q;
  };
  uint8_t* xcodes = take((size_t)kMaxF4Tokens * d / 2);
  uint8_t* xscales = take(f4_scale_bytes(d));
  float* sx = (float*)take(kMaxF4Tokens * 4);
  uint8_t* sfe = take(nvf4_sf_tile_bytes(V, d, A_KMAJOR));
  void* lmf = take(lmhead_fused_scratch_bytes(V, d));
  // the status word, and the token codes and scales of the rows past B (read by the MMA, their
  // columns dropped), start at zero
  CU(cudaMemsetAsync(base, 0, op_header() + align256((size_t)kMaxF4Tokens * d / 2) + align256(f4_scale_bytes(d)),
                     s));
  CU(nvf4_sf_tile(*E, nullptr, V, d, A_KMAJOR, sfe, s));
  ActQuantArgs q{};
  q.xf = d_x;
  q.K = d;
  q.codes = xcodes;
  q.scales = xscales;
  q.sx = sx;
  CU_LAUNCH(launch_k(k_act_quant, dim3(B), dim3(256), 0, s, q));
  char msg[256];
  CU(lmhead_fused_f4_launch(*E, sfe, xcodes, kMaxF4Tokens, 0, xscales, sx, B, V, d, mask_id, stats, d_s, lmf,
                            (int*)base, s, msg, sizeof(msg)));
  return DLM_OK;
}

static bool moe_shape_ok(int d, const dlm_moe_weights* w) {
  if (!w) return false;
  const long EF = (long)w->n_experts * w->ffn_expert;
  return w->n_experts >= 1 && w->n_experts <= 256 && w->top_k >= 1 && w->top_k <= 8 &&
         w->top_k <= w->n_experts && w->ffn_expert >= 64 && w->ffn_expert % 64 == 0 && EF % 256 == 0 &&
         EF <= 65536 && d >= 256 && d % 256 == 0 && d <= 8192;
}
static size_t moe_tile_bytes_pair(int d, const dlm_moe_weights* w) {
  return align256(nvf4_sf_tile_bytes(w->n_experts * w->ffn_expert, d, A_PAIR));
}

size_t dlm_moe_prepare_size(int d, const dlm_moe_weights* w) {
  if (!moe_shape_ok(d, w)) return 0;
  const int EF = w->n_experts * w->ffn_expert;
  return moe_tile_bytes_pair(d, w) + align256(nvf4_sf_tile_bytes(d, EF, A_KMAJOR));
}

dlm_status dlm_moe_prepare(int d, const dlm_moe_weights* w, void* d_tiles, size_t bytes, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!w || !d_tiles || !w->q_gate.scales || !w->q_up.scales || !w->q_down.scales) return DLM_EINVAL;
  if (!moe_shape_ok(d, w)) return DLM_EUNSUPPORTED;
  if (bytes < dlm_moe_prepare_size(d, w)) return DLM_ENOMEM_WS;
  cudaStream_t s = (cudaStream_t)stream;
  const int EF = w->n_experts * w->ffn_expert;
  uint8_t* base = (uint8_t*)d_tiles;
  CU(nvf4_sf_tile(w->q_gate, &w->q_up, EF, d, A_PAIR, base, s));
  CU(nvf4_sf_tile(w->q_down, nullptr, d, EF, A_KMAJOR, base + moe_tile_bytes_pair(d, w), s));
  return DLM_OK;
}

static size_t moe_partial_bytes(int T, int d, int EF) {
  const size_t a = gemm_fp4_partial_bytes(T, EF, d, A_PAIR), b = gemm_fp4_partial_bytes(T, d, EF, A_KMAJOR);
  return a > b ? a : b;
}

size_t dlm_moe_scratch_size(int T, int d, const dlm_moe_weights* w) {
  if (T < 1 || T > kMaxF4Tokens || !moe_shape_ok(d, w)) return 0;
  const int E = w->n_experts, EF = E * w->ffn_expert, K = EF > d ? EF : d;
  return op_header() + op_counters(K) + align256(moe_partial_bytes(T, d, EF)) +
         align256((size_t)kMaxF4Tokens * K / 2) + align256(f4_scale_bytes(K)) + align256(kMaxF4Tokens * 4) +
         align256((size_t)T * d * 4) + 2 * align256((size_t)T * E * 4) + 2 * align256((size_t)T * EF * 2) +
         align256((size_t)(EF / 64) * T * 4);
}

dlm_status dlm_moe_mlp_nvfp4(const float* d_h_in, float* d_h_out, int T, int d, float rms_eps,
                             const dlm_moe_weights* w, const void* d_tiles, int32_t* d_topk_idx, float* d_topk_w,
                             void* d_scratch, size_t scratch_bytes, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_h_in || !d_h_out || d_h_in == d_h_out || !w || !d_tiles || !d_scratch || !w->w_router ||
      !w->mlp_norm || !w->q_gate.codes || !w->q_up.codes || !w->q_down.codes || !std::isfinite(rms_eps) ||
      T < 1 || !std::isfinite(w->q_gate.tensor_scale) || !std::isfinite(w->q_up.tensor_scale) ||
      !std::isfinite(w->q_down.tensor_scale))
    return DLM_EINVAL;
  if (T > kMaxF4Tokens || !moe_shape_ok(d, w)) return DLM_EUNSUPPORTED;
  if (scratch_bytes < dlm_moe_scratch_size(T, d, w)) return DLM_ENOMEM_WS;
  CU((cudaError_t)gemm_fp4_init_attributes());
  cudaStream_t s = (cudaStream_t)stream;
  const int E = w->n_experts, F = w->ffn_expert, EF = E * F, K = EF > d ? EF : d;
  OpScratch sc(d_scratch, K, moe_partial_bytes(T, d, EF));
  uint8_t* xcodes = sc.take<uint8_t>((size_t)kMaxF4Tokens * K / 2);
  uint8_t* xscales = sc.take<uint8_t>(f4_scale_bytes(K));
  float* sx = sc.take<float>(kMaxF4Tokens);
  float* x = sc.take<float>((size_t)T * d);
  float* logits = sc.take<float>((size_t)T * E);
  float* route_w = sc.take<float>((size_t)T * E);
  __nv_bfloat16* act = sc.take<__nv_bfloat16>((size_t)2 * T * EF);  // high halves, then low halves
  float* act_amax = sc.take<float>((size_t)(EF / 64) * T);
  // the status word, and the token codes and scales of the rows past T (read by the MMA,
  // their columns dropped), start at zero
  CU(cudaMemsetAsync(d_scratch, 0, op_header(), s));
  CU(cudaMemsetAsync(xcodes, 0, (size_t)kMaxF4Tokens * K / 2, s));
  CU(cudaMemsetAsync(xscales, 0, f4_scale_bytes(K), s));
  MoeRouteArgs ra{};
  ra.h = d_h_in;
  ra.g = (const __nv_bfloat16*)w->mlp_norm;
  ra.wr = (const __nv_bfloat16*)w->w_router;
  ra.eps = rms_eps;
  ra.T = T;
  ra.d = d;
  ra.E = E;
  ra.k = w->top_k;
  ra.x = x;
  ra.logits = logits;
  ra.route_w = route_w;
  ra.topk_idx = d_topk_idx;
  ra.topk_w = d_topk_w;
  CU_LAUNCH(launch_k(k_moe_logits, dim3(T, (E + 7) / 8), dim3(256), d * 4, s, ra));
  CU_LAUNCH(launch_k(k_moe_topk, dim3((T + 7) / 8), dim3(256), 0, s, ra));
  ActQuantArgs q{};
  q.xf = x;
  q.K = d;
  q.codes = xcodes;
  q.scales = xscales;
  q.sx = sx;
  CU_LAUNCH(launch_k(k_act_quant, dim3(T), dim3(256), 0, s, q));
  const uint8_t* tiles = (const uint8_t*)d_tiles;
  char msg[256];
  GemmF4Plan p;
  // every expert's gate/up rows on every row of x
  if (!gemm_fp4_plan(&p, A_PAIR, w->q_gate, &w->q_up, tiles, xcodes, xscales, kMaxF4Tokens, sx, T, EF, d, sc.partial,
                     msg, sizeof(msg)))
    return DLM_EUNSUPPORTED;
  CU(gemm_fp4_launch(p, sc.err, s));
  EpiArgs es{};
  es.op = EPI_SILU;
  es.act = act;
  es.act_lo = (long)T * EF;
  es.act_amax = act_amax;
  es.route_w = route_w;
  es.route_e = E;
  es.route_f = F;
  {
    FinishArgs fa{p.out, es, EF};
    CU_LAUNCH(launch_k(k_finish_silu, dim3(p.out.n_tiles, (T + 31) / 32), dim3(256), 0, s, fa));
  }
  // the weighted expert activations, one row of E F per token, quantized per row
  ActQuantArgs qa{};
  qa.xb = act;
  qa.xb_lo = (long)T * EF;
  qa.K = EF;
  qa.codes = xcodes;
  qa.scales = xscales;
  qa.sx = sx;
  qa.amax = act_amax;
  qa.n_amax = EF / 64;
  qa.T = T;
  CU_LAUNCH(launch_k(k_act_quant_wide, dim3((unsigned)((EF / 16 + 255) / 256), T), dim3(256), 0, s, qa));
  if (!gemm_fp4_plan(&p, A_KMAJOR, w->q_down, nullptr, tiles + moe_tile_bytes_pair(d, w), xcodes, xscales,
                     kMaxF4Tokens, sx, T, d, EF, sc.partial, msg, sizeof(msg)))
    return DLM_EUNSUPPORTED;
  CU(gemm_fp4_launch(p, sc.err, s));
  EpiArgs eo{};
  eo.op = EPI_STORE;
  eo.out = d_h_out;
  eo.ld = d;
  eo.add = d_h_in;
  FinishArgs fo{p.out, eo, d};
  CU_LAUNCH(launch_k(k_finish_store, dim3(p.out.n_tiles, T), dim3(kTileM), 0, s, fo));
  return DLM_OK;
}

size_t dlm_gemm_nvfp4_scratch_size(int T, int N, int K) {
  if (T < 1 || T > kMaxF4Tokens || N < 1 || K < 256 || K % 256 || K > 16384) return 0;
  return op_header() + op_counters(N) + align256(gemm_fp4_partial_bytes(T, N, K, A_KMAJOR)) +
         align256((size_t)kMaxF4Tokens * K / 2) + align256(f4_scale_bytes(K)) + align256(kMaxF4Tokens * 4) +
         align256(nvf4_sf_tile_bytes(N, K, A_KMAJOR));
}

dlm_status dlm_gemm_nvfp4(const float* d_x, const dlm_nvfp4_matrix* w, float* d_y, int T, int N, int K,
                          void* d_scratch, size_t scratch_bytes, void* stream) {
  dlm_ctx* ctx = nullptr;
  if (!d_x || !w || !w->codes || !w->scales || !d_scratch || T < 1 || T > kMaxF4Tokens || N < 1 || K < 256 ||
      K % 256 || K > 16384)
    return DLM_EINVAL;
  if (scratch_bytes < dlm_gemm_nvfp4_scratch_size(T, N, K)) return DLM_ENOMEM_WS;
  CU((cudaError_t)gemm_fp4_init_attributes());
  cudaStream_t s = (cudaStream_t)stream;
  OpScratch sc(d_scratch, N, gemm_fp4_partial_bytes(T, N, K, A_KMAJOR));
  uint8_t* xcodes = sc.take<uint8_t>((size_t)kMaxF4Tokens * K / 2);
  uint8_t* xscales = sc.take<uint8_t>(f4_scale_bytes(K));
  float* sx = sc.take<float>(kMaxF4Tokens);
  uint8_t* sfa = sc.take<uint8_t>(nvf4_sf_tile_bytes(N, K, A_KMAJOR));
  CU(cudaMemsetAsync(d_scratch, 0, op_header(), s));
  // rows T.. of the token codes and scales are read by the MMA (their columns are dropped)
  CU(cudaMemsetAsync(xcodes, 0, (size_t)kMaxF4Tokens * K / 2, s));
  CU(cudaMemsetAsync(xscales, 0, f4_scale_bytes(K), s));
  CU(nvf4_sf_tile(*w, nullptr, N, K, A_KMAJOR, sfa, s));
  ActQuantArgs q{};
  q.xf = d_x;
  q.K = K;
  q.codes = xcodes;
  q.scales = xscales;
  q.sx = sx;
  CU_LAUNCH(launch_k(k_act_quant, dim3(T), dim3(256), 0, s, q));
  char msg[256];
  GemmF4Plan p;
  if (!gemm_fp4_plan(&p, A_KMAJOR, *w, nullptr, sfa, xcodes, xscales, kMaxF4Tokens, sx, T, N, K, sc.partial, msg,
                     sizeof(msg)))
    return DLM_EUNSUPPORTED;
  CU(gemm_fp4_launch(p, sc.err, s));
  if (d_y) {
    EpiArgs e{};
    e.op = EPI_STORE;
    e.out = d_y;
    e.ld = N;
    FinishArgs fa{p.out, e, N};
    CU_LAUNCH(launch_k(k_finish_store, dim3(p.out.n_tiles, T), dim3(kTileM), 0, s, fa));
  }
  return DLM_OK;
}

}  // extern "C"

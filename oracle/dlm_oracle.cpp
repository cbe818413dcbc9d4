// dlm_oracle.cpp -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, obviously-correct CPU restatement (C++17, fp64 arithmetic) of one
// residual block-diffusion denoising round and the loop around it.  It exists to
// check the CUDA path; only tests/, __graft_entry__.smoke() and bench.py's
// cpu_baseline / reference leg may load it.  It shares no code, header, table or
// helper with the CUDA library and includes nothing from it.
//
// Sources (cited by page title and section):
//   [blog]  "ORL: diffusion LLMs get a learnable 'tokens per forward' -- 2,788 tok/s on
//           one RTX 5090, 7,708 on 8x B200" (richland.au), section "What shipped":
//             - opening paragraph: blocks are decoded by denoising rounds; each round gives a
//               distribution over the still-unresolved tokens; the block commits after
//               enough rounds.
//             - "On-policy residual learning": the previous round's distribution is fed back
//               into the next round through a self-conditioning adapter on the tied embedding.
//             - "Adjacent entropy contraction": more positions clear the commit bar each round.
//             - "dlmrt, the inference engine": one CUDA graph per block, a conditional node
//               decides after every round whether to continue.
//   [card]  "QwenDLM-4B-ORL" model card (shadowgraph.io), section "The paper's evaluation
//           pipeline": serve flags SDAR_FUSED_ROW_STATS=1 (LM head fused with per-row
//           statistics), SDAR_COMMIT_GRAPH=1 (commit inside the graph), --dllm-algorithm
//           SDARPrefixKV (block decoding over a prefix KV cache).
//   [news]  "ORL 与 dlmrt 开源" (openai-hub.com), section "dLLM 是什么": positions are
//           predicted in parallel and revised according to confidence.
//
// Where the pages leave a step open the oracle takes these readings (each is listed with
// its reason in the design notes of the repository):
//   R1 adapter: h0_i = E[x_i] + W_a * s_i, W_a is d x d (out x in), no bias / norm / gate.
//   R2 residual rows: s_i = P_prev,i @ E only for positions still uncommitted that were
//      predicted in the previous round; round 0 and committed positions have s_i = 0.
//   R3 mask token: mask_id (normally V-1) is embedded through its own row of E and is
//      excluded (logit -inf) from the softmax / argmax of the decode path; mask_id < 0
//      turns the exclusion off.
//   R4 commit: threshold mode commits every uncommitted i with maxprob_i >= tau, and if
//      none qualifies the single uncommitted i with the largest maxprob (ties -> lowest i);
//      fixed-k mode commits the top min(k, remaining) by maxprob (ties -> lowest i).
//      A committed token is the row argmax (ties -> lowest vocab id).  No remasking.
//   R5 KV for a committed block: one clean forward (committed tokens, s = 0, no LM head)
//      writes its K/V rows; the prompt is prefilled with a plain causal forward.
//   R6 architecture: pre-norm transformer, RMSNorm(v) = v / sqrt(mean(v^2) + eps) * g,
//      NeoX rotate-half RoPE with theta_j = base^(-2j/hd) at absolute positions,
//      GQA (q head h reads kv head floor(h * Hkv / Hq)), softmax(q.k / sqrt(hd)),
//      SiLU-gated MLP, no biases, tied LM head (logits = RMSNorm(h) E^T).
//   R7 entropy in nats; maxprob = exp(m - lse).
//   R8 NVFP4: per-tensor fp32 scale S = amax / (6 * 448); per 16-element block an e4m3
//      scale sigma = RNE_e4m3(amax_blk / (6 S)); code q = RNE onto the e2m1 grid of
//      w / (sigma S), saturating at +-6; dequant = q * sigma * S.  Activations use the
//      same quantizer with one fp32 scale per row.
//   R9 attention operand precision (option act_round): the KV cache holds bf16 values and
//      the attention takes bf16 queries, so with act_round set the oracle rounds q, k and v
//      to bf16 (round-to-nearest-even) after RoPE, as they are stored; integer decisions
//      are then taken on the same attention operands.  Every other value stays fp64.
//   R13 FP8 KV cache (option kv_fp8; [blog] "What shipped", "dlmrt, the inference engine":
//      the KV cache is FP8): every K and V row of hd values (one layer, one KV head, one
//      position) is stored as OCP e4m3 codes with one fp32 scale s = amax(|row|) / 448, code =
//      RNE_e4m3(x / s) saturating at 448, value = e4m3(code) * s.  q stays bf16 (R9); the K
//      and V rows are quantized from their unrounded values.
//   R14 routed-expert MLP ([blog] "What shipped", "dlmrt, the inference engine": routed
//      experts run NVFP4 on FP4 tensor cores; the pages give neither the routing rule nor
//      the expert shapes, so this is the plainest reading): x = RMSNorm(h) g; router logits
//      l = x W_r^T (W_r bf16 [E][d]); p = softmax(l) over the E experts; the k experts of
//      largest p are selected (ties to the lower index) with weights w_e = p_e / sum of the
//      selected p; every expert is a SiLU-gated MLP (gate, up [F][d], down [d][F]) and the
//      sub-block adds h += sum_e w_e down_e(silu(gate_e x) * up_e x).  The experts' gate and
//      up matrices are stacked along rows ([E F][d], expert e in rows [e F, (e + 1) F)) and
//      their down matrices side by side along columns ([d][E F]), one NVFP4 tensor scale
//      each; the activation row entering the down projection is the concatenation over the
//      experts of w_e silu(.) * up(.) (zeros for the experts not selected), quantized per
//      row like every NVFP4 GEMM input (R8), so the weighted sum over the experts is one
//      contraction over E F.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- number formats
double bf16_to_double(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

// Round a double to the nearest bf16 value (ties to even), returned as a double.
// bf16: 8 significant bits, exponent range of fp32, subnormal quantum 2^-133.
double round_bf16(double x) {
  if (!std::isfinite(x) || x == 0.0) return x;
  int e;
  std::frexp(x, &e);                 // |x| = f * 2^e, f in [0.5, 1)
  int qexp = e - 8;                  // quantum for 8 significant bits
  if (qexp < -133) qexp = -133;      // subnormal range
  double q = std::ldexp(1.0, qexp);
  double r = std::nearbyint(x / q) * q;  // default rounding mode: ties to even
  const double maxv = std::ldexp(255.0, 127 - 7);  // largest finite bf16
  if (std::fabs(r) > maxv) return std::copysign(std::numeric_limits<double>::infinity(), x);
  return r;
}

// OCP E4M3 (fn variant): bias 7, 3 mantissa bits, max 448, subnormal quantum 2^-9.
// Round-to-nearest-even of a non-negative fp32 value, saturating at 448 (scales are >= 0).
double round_e4m3_nonneg(float xf) {
  double x = double(xf);
  if (!(x > 0.0)) return 0.0;
  int e;
  std::frexp(x, &e);
  int qexp = e - 4;                  // 4 significant bits
  if (qexp < -9) qexp = -9;
  double q = std::ldexp(1.0, qexp);
  double r = std::nearbyint(x / q) * q;
  if (r > 448.0) r = 448.0;
  return r;
}

// e4m3 bit pattern of a representable non-negative value.
uint8_t e4m3_bits(double v) {
  if (v == 0.0) return 0;
  int e;
  double f = std::frexp(v, &e);      // v = f 2^e, f in [0.5,1)
  int E = e - 1 + 7;                 // biased exponent of 1.m form
  if (E <= 0) {                      // subnormal: v = m * 2^-9
    int m = int(std::lround(v / std::ldexp(1.0, -9)));
    return uint8_t(m & 7);
  }
  int m = int(std::lround((f * 2.0 - 1.0) * 8.0));
  return uint8_t((E << 3) | m);
}

double e4m3_value(uint8_t b) {
  int E = (b >> 3) & 15, m = b & 7;
  if (E == 0) return std::ldexp(double(m), -9);
  return std::ldexp(1.0 + m / 8.0, E - 7);
}

// e2m1 magnitudes indexed by the 3 low code bits.
const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

// Round-to-nearest-even onto the e2m1 grid (ties go to the even code), saturating at 6.
uint8_t e2m1_encode(float rf) {
  double r = double(rf);
  uint8_t sign = (r < 0.0) ? 8 : 0;
  double a = std::fabs(r);
  if (!(a == a)) return sign;        // NaN never occurs for finite inputs
  if (a >= 6.0) return uint8_t(sign | 7);
  int best = 0;
  for (int c = 1; c < 8; ++c) {
    double dc = std::fabs(a - kE2M1[c]), db = std::fabs(a - kE2M1[best]);
    if (dc < db || (dc == db && (c % 2 == 0) && (best % 2 == 1))) best = c;
  }
  return uint8_t(sign | best);
}

// Margin of a rounding decision: the distance of the rounded quantity from its nearest
// decision boundary, relative to the boundary.  Quantization codes are integer decisions
// taken from floats; two computations whose inputs differ by a relative epsilon can round
// differently only where this margin is below about epsilon (like a top-2 logit gap for
// an argmax).
double e2m1_margin(float rf) {
  const double a = std::fabs(double(rf));
  const double bounds[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};  // midpoints of kE2M1
  double m = std::numeric_limits<double>::infinity();
  for (double b : bounds) m = std::min(m, std::fabs(a - b) / b);
  return m;
}

// Margin of round_e4m3_nonneg(x): the midpoints between neighbouring e4m3 values inside
// x's binade are (k + 1/2) q (q = the binade's spacing), and the one just below the binade
// lies a quarter spacing under its lower edge; values from 448 up saturate to 448.
double e4m3_margin(float xf) {
  const double x = double(xf);
  if (!(x > 0.0)) return std::numeric_limits<double>::infinity();
  if (x >= 448.0) return (x - 432.0) / 432.0;  // saturated: 432 is the midpoint below 448
  int e;
  std::frexp(x, &e);
  int qexp = e - 4;
  if (qexp < -9) qexp = -9;
  const double q = std::ldexp(1.0, qexp);
  const double mid = (std::floor(x / q) + 0.5) * q;
  double m = std::fabs(x - mid) / mid;
  if (e - 4 >= -9) {
    const double below = std::ldexp(1.0, e - 1) - q / 4;
    m = std::min(m, std::fabs(x - below) / below);
  }
  return m;
}

double e2m1_value(uint8_t c) {
  double v = kE2M1[c & 7];
  return (c & 8) ? -v : v;
}

// ---------------------------------------------------------------- parallel helper
int g_threads = 0;  // 0 = hardware concurrency

// Runs f(i) for i in [0, n) over a fixed contiguous partition; every i is computed by
// exactly one thread in a fixed order, so results do not depend on the thread count.
template <class F>
void parallel_for(long n, F f) {
  int nt = g_threads > 0 ? g_threads : int(std::thread::hardware_concurrency());
  if (nt < 1) nt = 1;
  if (n < 64 || nt == 1) {
    for (long i = 0; i < n; ++i) f(i);
    return;
  }
  if (nt > n) nt = int(n);
  std::vector<std::thread> th;
  for (int t = 0; t < nt; ++t) {
    long a = n * t / nt, b = n * (t + 1) / nt;
    th.emplace_back([=, &f] { for (long i = a; i < b; ++i) f(i); });
  }
  for (auto& x : th) x.join();
}

// Quantize one row of `cols` values (cols % 16 == 0) with tensor scale S; `margin`
// (optional) is lowered to the smallest margin of the row's rounding decisions.
void quantize_row(const float* w, int cols, float S, uint8_t* codes, uint8_t* scales, double* margin) {
  for (int b = 0; b < cols / 16; ++b) {
    float amax = 0.0f;
    for (int j = 0; j < 16; ++j) amax = std::max(amax, std::fabs(w[b * 16 + j]));
    double sig = 0.0;
    if (S > 0.0f) {
      sig = round_e4m3_nonneg(amax / (6.0f * S));
      if (margin) *margin = std::min(*margin, e4m3_margin(amax / (6.0f * S)));
    }
    scales[b] = e4m3_bits(sig);
    float denom = float(sig) * S;
    for (int j = 0; j < 16; ++j) {
      uint8_t c = 0;
      if (denom > 0.0f) {
        c = e2m1_encode(w[b * 16 + j] / denom);
        if (margin) *margin = std::min(*margin, e2m1_margin(w[b * 16 + j] / denom));
      }
      int idx = b * 16 + j;
      if (idx % 2 == 0) codes[idx / 2] = c;
      else codes[idx / 2] = uint8_t(codes[idx / 2] | (c << 4));
    }
  }
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------- public structs
// A weight matrix W[rows][cols] (out x in, row-major).  Either bf16 bits (fmt 0) or
// NVFP4 (fmt 1): codes[rows][cols/2] (element 2j in the low nibble), scales[rows][cols/16]
// (e4m3 bits) and one fp32 tensor scale.
typedef struct orc_mat {
  int fmt;
  int rows, cols;
  const uint16_t* bf16;
  const uint8_t* codes;
  const uint8_t* scales;
  float tscale;
} orc_mat;

typedef struct orc_cfg {
  int n_layers, d, n_q_heads, n_kv_heads, head_dim, ffn, vocab, mask_id, block_size;
  double rope_theta, rms_eps;
  int act_round;      // R9
  int act_fp4;        // NVFP4 GEMMs quantize their input rows (R8); 0 for bf16 models
  int kv_fp8;         // R13
} orc_cfg;

typedef struct orc_layer {
  const uint16_t* attn_norm;  // [d] bf16
  orc_mat w_qkv;              // [(Hq + 2 Hkv) hd][d]; rows: q heads, then k heads, then v heads
  orc_mat w_o;                // [d][Hq hd]
  const uint16_t* mlp_norm;   // [d]
  orc_mat w_gate, w_up;       // [F][d]
  orc_mat w_down;             // [d][F]
} orc_layer;

typedef struct orc_model {
  orc_mat embed;              // E [V][d], tied LM head
  orc_mat w_adapter;          // W_a [d][d]
  const uint16_t* final_norm; // [d]
  const orc_layer* layers;    // [n_layers]
} orc_model;

// KV cache owned by the caller: k, v = [n_layers][n_kv_heads][max_ctx][head_dim] doubles.
typedef struct orc_kv {
  int max_ctx;
  double* k;
  double* v;
} orc_kv;

// Per-row statistics of one row of logits (R7).
typedef struct orc_stats {
  double m, lse, maxprob, entropy;
  int argmax;
  double gap2;     // largest minus second-largest logit (ambiguity of the argmax)
  double qmargin;  // smallest margin of the row's NVFP4 activation rounding decisions
                   // (e2m1_margin / e4m3_margin) in the forward pass; +inf without any
} orc_stats;

// FP8 KV row (R13): n values -> e4m3 codes and one fp32 scale amax / 448; `out` (optional)
// receives the stored values e4m3(code) * scale.  Returns the scale.
float orc_kv_quantize_row(const double* x, int n, uint8_t* codes, double* out) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(float(x[i])));
  const float s = amax / 448.0f;
  for (int i = 0; i < n; ++i) {
    double v = 0.0;
    uint8_t c = 0;
    if (s > 0.0f) {
      const float r = float(x[i]) / s;
      const double q = round_e4m3_nonneg(std::fabs(r));  // magnitude, RNE, saturating
      c = uint8_t(e4m3_bits(q) | (r < 0.0f ? 0x80 : 0));
      v = (r < 0.0f ? -q : q) * double(s);
    }
    if (codes) codes[i] = c;
    if (out) out[i] = v;
  }
  return s;
}

void orc_set_threads(int n) { g_threads = n; }
int orc_hw_threads(void) { return int(std::thread::hardware_concurrency()); }

double orc_round_bf16(double x) { return round_bf16(x); }

// ---------------------------------------------------------------- NVFP4 codec (R8)
float orc_nvfp4_tensor_scale(const float* w, long n) {
  float amax = 0.0f;
  for (long i = 0; i < n; ++i) amax = std::max(amax, std::fabs(w[i]));
  return amax / (6.0f * 448.0f);
}

// Quantize one row of `cols` values (cols % 16 == 0) with tensor scale S.
void orc_nvfp4_quantize_row(const float* w, int cols, float S, uint8_t* codes, uint8_t* scales) {
  quantize_row(w, cols, S, codes, scales, nullptr);
}

void orc_nvfp4_quantize(const float* w, int rows, int cols, uint8_t* codes, uint8_t* scales,
                        float* tscale) {
  float S = orc_nvfp4_tensor_scale(w, long(rows) * cols);
  *tscale = S;
  parallel_for(rows, [&](long r) {
    orc_nvfp4_quantize_row(w + r * long(cols), cols, S, codes + r * long(cols / 2),
                           scales + r * long(cols / 16));
  });
}

double orc_nvfp4_value(const uint8_t* codes, const uint8_t* scales, float S, long row_elems,
                       long r, long c) {
  uint8_t byte = codes[(r * row_elems + c) / 2];
  uint8_t code = (c % 2 == 0) ? (byte & 15) : (byte >> 4);
  double sig = e4m3_value(scales[(r * row_elems + c) / 16]);
  return double(float(float(e2m1_value(code) * sig) * S));
}

void orc_nvfp4_dequant(const uint8_t* codes, const uint8_t* scales, float S, int rows, int cols,
                       double* out) {
  for (long r = 0; r < rows; ++r)
    for (long c = 0; c < cols; ++c) out[r * cols + c] = orc_nvfp4_value(codes, scales, S, cols, r, c);
}

double orc_e2m1_value(int code) { return e2m1_value(uint8_t(code)); }
int orc_e2m1_encode(float r) { return e2m1_encode(r); }
double orc_e4m3_round(float x) { return round_e4m3_nonneg(x); }
int orc_e4m3_bits(double v) { return e4m3_bits(v); }
double orc_e4m3_value(int b) { return e4m3_value(uint8_t(b)); }

}  // extern "C"

namespace {

// Row r of a weight matrix as doubles.
void mat_row(const orc_mat& W, long r, double* out) {
  if (W.fmt == 0) {
    const uint16_t* p = W.bf16 + r * long(W.cols);
    for (int c = 0; c < W.cols; ++c) out[c] = bf16_to_double(p[c]);
  } else {
    for (int c = 0; c < W.cols; ++c) out[c] = orc_nvfp4_value(W.codes, W.scales, W.tscale, W.cols, r, c);
  }
}

// NVFP4 input quantization of one activation row (R8): per-row fp32 scale.  `margin`
// (optional) is lowered to the smallest margin of the row's rounding decisions.
void quantize_act_row(const double* x, int cols, double* out, double* margin) {
  std::vector<float> xf(cols);
  for (int i = 0; i < cols; ++i) xf[i] = float(x[i]);
  float S = orc_nvfp4_tensor_scale(xf.data(), cols);
  std::vector<uint8_t> codes(cols / 2), scales(cols / 16);
  quantize_row(xf.data(), cols, S, codes.data(), scales.data(), margin);
  for (int c = 0; c < cols; ++c) out[c] = orc_nvfp4_value(codes.data(), scales.data(), S, cols, 0, c);
}

// y[t][n] = sum_k x[t][k] W[n][k]  (plain triple loop, fp64).  qm[t] (optional) collects
// the rounding margins of row t's input quantization.
void linear(const double* x, int T, const orc_mat& W, double* y, bool act_fp4, double* qm = nullptr) {
  const int K = W.cols, N = W.rows;
  std::vector<double> xq;
  const double* xin = x;
  if (act_fp4 && W.fmt == 1) {
    xq.resize(size_t(T) * K);
    for (int t = 0; t < T; ++t)
      quantize_act_row(x + size_t(t) * K, K, xq.data() + size_t(t) * K, qm ? qm + t : nullptr);
    xin = xq.data();
  }
  // x transposed to [K][T] so that the T sums of one weight row advance together; every
  // output is still the plain sum over k = 0 .. K-1 in ascending order.
  std::vector<double> xt(size_t(K) * T);
  for (int t = 0; t < T; ++t)
    for (int k = 0; k < K; ++k) xt[size_t(k) * T + t] = xin[size_t(t) * K + k];
  parallel_for(N, [&](long n) {
    std::vector<double> w(K), acc(T, 0.0);
    mat_row(W, n, w.data());
    for (int k = 0; k < K; ++k) {
      const double wk = w[k];
      const double* xk = xt.data() + size_t(k) * T;
      for (int t = 0; t < T; ++t) acc[t] += xk[t] * wk;
    }
    for (int t = 0; t < T; ++t) y[size_t(t) * N + n] = acc[t];
  });
}

void rmsnorm(const double* x, int n, const uint16_t* g, double eps, double* out) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double r = 1.0 / std::sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) out[i] = x[i] * r * bf16_to_double(g[i]);
}

void rope(double* x, int hd, long pos, double base) {
  const int half = hd / 2;
  for (int j = 0; j < half; ++j) {
    double theta = std::pow(base, -2.0 * j / hd);
    double a = double(pos) * theta;
    double c = std::cos(a), s = std::sin(a);
    double x0 = x[j], x1 = x[j + half];
    x[j] = x0 * c - x1 * s;
    x[j + half] = x0 * s + x1 * c;
  }
}

inline double maybe_round(double v, bool on) { return on ? round_bf16(v) : v; }

}  // namespace

extern "C" {

void orc_linear(const double* x, int T, const orc_mat* W, double* y, int act_fp4) {
  linear(x, T, *W, y, act_fp4 != 0);
}

void orc_rmsnorm(const double* x, int rows, int n, const uint16_t* g, double eps, double* out) {
  for (int r = 0; r < rows; ++r) rmsnorm(x + size_t(r) * n, n, g, eps, out + size_t(r) * n);
}

void orc_rope(double* x, int hd, long pos, double base) { rope(x, hd, pos, base); }

// Block-diffusion attention for nq query positions pos0 .. pos0+nq-1 of one layer.
//   q      [nq][Hq][hd]
//   kc, vc [Hkv][max_ctx][hd] (keys/values at absolute positions; rows [0, pos0+nq) valid)
//   out    [nq][Hq][hd]
// causal == 0: every query sees keys [0, pos0 + nq) (prefix causal, block bidirectional).
// causal != 0: query at position p sees keys [0, p].
void orc_attention(const double* q, int nq, int Hq, int Hkv, int hd, const double* kc,
                   const double* vc, int max_ctx, int pos0, int causal, double* out) {
  const double scale = 1.0 / std::sqrt(double(hd));
  parallel_for(long(nq) * Hq, [&](long idx) {
    int i = int(idx / Hq), h = int(idx % Hq);
    int g = int(long(h) * Hkv / Hq);
    int nkeys = causal ? (pos0 + i + 1) : (pos0 + nq);
    const double* qi = q + (size_t(i) * Hq + h) * hd;
    std::vector<double> sc(nkeys);
    double m = -std::numeric_limits<double>::infinity();
    for (int j = 0; j < nkeys; ++j) {
      const double* kj = kc + (size_t(g) * max_ctx + j) * hd;
      double a = 0.0;
      for (int e = 0; e < hd; ++e) a += qi[e] * kj[e];
      sc[j] = a * scale;
      m = std::max(m, sc[j]);
    }
    double z = 0.0;
    for (int j = 0; j < nkeys; ++j) { sc[j] = std::exp(sc[j] - m); z += sc[j]; }
    double* oi = out + (size_t(i) * Hq + h) * hd;
    for (int e = 0; e < hd; ++e) oi[e] = 0.0;
    for (int j = 0; j < nkeys; ++j) {
      const double* vj = vc + (size_t(g) * max_ctx + j) * hd;
      double p = sc[j] / z;
      for (int e = 0; e < hd; ++e) oi[e] += p * vj[e];
    }
  });
}

// Row statistics of logits[B][V] (R3, R7), straight from the definitions:
// p = softmax(l) over the non-excluded ids, maxprob = max p, argmax = first index of the
// max logit, entropy = -sum p ln p.
void orc_rowstats(const double* logits, int B, int V, int mask_id, orc_stats* st) {
  for (int b = 0; b < B; ++b) {
    const double* l = logits + size_t(b) * V;
    double m = -std::numeric_limits<double>::infinity();
    int am = -1;
    for (int v = 0; v < V; ++v) {
      if (v == mask_id) continue;
      if (l[v] > m) { m = l[v]; am = v; }
    }
    double z = 0.0;
    for (int v = 0; v < V; ++v) if (v != mask_id) z += std::exp(l[v] - m);
    double lse = m + std::log(z);
    double H = 0.0;
    for (int v = 0; v < V; ++v) {
      if (v == mask_id) continue;
      double lp = l[v] - lse;
      double p = std::exp(lp);
      if (p > 0.0) H -= p * lp;
    }
    double second = -std::numeric_limits<double>::infinity();
    for (int v = 0; v < V; ++v)
      if (v != mask_id && v != am) second = std::max(second, l[v]);
    st[b].gap2 = m - second;
    st[b].qmargin = std::numeric_limits<double>::infinity();
    st[b].m = m;
    st[b].lse = lse;
    st[b].maxprob = std::exp(m - lse);
    st[b].entropy = H;
    st[b].argmax = am;
  }
}

// Routed-expert MLP sub-block (R14).  h_in, h_out [T][d]; logits [T][E] (optional);
// topk_idx, topk_w [T][k]; qmargin [T] (optional, act_fp4 only: the smallest distance of an
// activation to a quantization decision boundary, as orc_lmhead reports it).
typedef struct orc_moe {
  int n_experts, top_k, ffn_expert;
  const uint16_t* w_router;  // bf16 [E][d]
  const uint16_t* norm;      // bf16 [d]
  orc_mat gate, up;          // [E F][d]
  orc_mat down;              // [d][E F]
} orc_moe;

void orc_moe_mlp(const double* h_in, int T, int d, double eps, const orc_moe* M, int act_fp4, double* h_out,
                 double* logits_out, int* topk_idx, double* topk_w, double* qmargin) {
  const int E = M->n_experts, k = M->top_k, F = M->ffn_expert, EF = E * F;
  const bool fp4 = act_fp4 != 0;
  std::vector<double> x(size_t(T) * d), l(size_t(T) * E), sel_w(size_t(T) * E, 0.0);
  std::vector<double> qm(T, std::numeric_limits<double>::infinity());
  for (int t = 0; t < T; ++t) rmsnorm(h_in + size_t(t) * d, d, M->norm, eps, x.data() + size_t(t) * d);
  for (int t = 0; t < T; ++t) {
    // router logits and softmax over all experts
    double mx = -std::numeric_limits<double>::infinity();
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += x[size_t(t) * d + c] * bf16_to_double(M->w_router[size_t(e) * d + c]);
      l[size_t(t) * E + e] = acc;
      mx = std::max(mx, acc);
    }
    std::vector<double> p(E);
    double z = 0.0;
    for (int e = 0; e < E; ++e) z += (p[e] = std::exp(l[size_t(t) * E + e] - mx));
    for (int e = 0; e < E; ++e) p[e] /= z;
    // top-k by probability, ties to the lower index; weights renormalised over the chosen
    std::vector<uint8_t> taken(E, 0);
    double zs = 0.0;
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || p[e] > p[best])) best = e;
      taken[best] = 1;
      topk_idx[size_t(t) * k + j] = best;
      zs += p[best];
    }
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[size_t(t) * k + j];
      topk_w[size_t(t) * k + j] = p[e] / zs;
      sel_w[size_t(t) * E + e] = p[e] / zs;
    }
  }
  if (logits_out) std::memcpy(logits_out, l.data(), l.size() * sizeof(double));
  // every expert on every row (the ones not selected get weight 0 below)
  std::vector<double> g(size_t(T) * EF), u(size_t(T) * EF), a(size_t(T) * EF), y(size_t(T) * d);
  linear(x.data(), T, M->gate, g.data(), fp4, qm.data());
  linear(x.data(), T, M->up, u.data(), fp4, qm.data());
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < EF; ++j) {
      const size_t i = size_t(t) * EF + j;
      const double w = sel_w[size_t(t) * E + j / F];
      a[i] = (w == 0.0) ? 0.0 : w * (g[i] / (1.0 + std::exp(-g[i]))) * u[i];
    }
  linear(a.data(), T, M->down, y.data(), fp4, qm.data());
  for (size_t i = 0; i < y.size(); ++i) h_out[i] = h_in[i] + y[i];
  if (qmargin)
    for (int t = 0; t < T; ++t) qmargin[t] = qm[t];
}

// Fused-LM-head semantics, computed plainly: logits = x E^T (x already normalised),
// row statistics, and s = P E where P = softmax(logits) (p_given == nullptr) or a given
// distribution p_given[B][V].  x[B][d]; s[B][d]; logits_out[B][V] optional.
void orc_lmhead(const double* x, int B, const orc_mat* E, int mask_id, int act_fp4,
                const double* p_given, orc_stats* st, double* s, double* logits_out) {
  const int V = E->rows, d = E->cols;
  std::vector<double> logits(size_t(B) * V), qm(B, std::numeric_limits<double>::infinity());
  linear(x, B, *E, logits.data(), act_fp4 != 0, qm.data());
  orc_rowstats(logits.data(), B, V, mask_id, st);
  for (int b = 0; b < B; ++b) st[b].qmargin = qm[b];
  if (logits_out) std::memcpy(logits_out, logits.data(), logits.size() * sizeof(double));
  std::vector<double> P(size_t(B) * V);
  for (int b = 0; b < B; ++b)
    for (int v = 0; v < V; ++v) {
      if (p_given) P[size_t(b) * V + v] = p_given[size_t(b) * V + v];
      else P[size_t(b) * V + v] = (v == mask_id) ? 0.0 : std::exp(logits[size_t(b) * V + v] - st[b].lse);
    }
  // s[b][c] = sum_v P[b][v] E[v][c]; parallel over columns c, each a plain V-sum.
  int nt = g_threads > 0 ? g_threads : int(std::thread::hardware_concurrency());
  if (nt < 1) nt = 1;
  std::vector<std::vector<double>> part(nt, std::vector<double>(size_t(B) * d, 0.0));
  // partition the vocabulary into nt contiguous ranges, then sum the ranges in order
  std::vector<std::thread> th;
  for (int t = 0; t < nt; ++t) {
    th.emplace_back([&, t] {
      long a = long(V) * t / nt, bnd = long(V) * (t + 1) / nt;
      std::vector<double> row(d);
      for (long v = a; v < bnd; ++v) {
        mat_row(*E, v, row.data());
        for (int b = 0; b < B; ++b) {
          double p = P[size_t(b) * V + v];
          if (p == 0.0) continue;
          double* sp = part[t].data() + size_t(b) * d;
          for (int c = 0; c < d; ++c) sp[c] += p * row[c];
        }
      }
    });
  }
  for (auto& x2 : th) x2.join();
  for (size_t i = 0; i < size_t(B) * d; ++i) {
    double acc = 0.0;
    for (int t = 0; t < nt; ++t) acc += part[t][i];
    s[i] = acc;
  }
}

// Commit rule (R4).  maxprob/argmax per position; tokens/committed updated in place.
// mode 0 = threshold tau with the min-1 rule, mode 1 = fixed top-k.  Returns the number
// of positions committed by this call.
int orc_commit(int B, const double* maxprob, const int* argmax, double tau, int mode, int k,
               int* tokens, uint8_t* committed) {
  std::vector<int> unc;
  for (int i = 0; i < B; ++i) if (!committed[i]) unc.push_back(i);
  if (unc.empty()) return 0;
  std::vector<int> sel;
  if (mode == 0) {
    for (int i : unc) if (maxprob[i] >= tau) sel.push_back(i);
    if (sel.empty()) {
      int best = unc[0];
      for (int i : unc) if (maxprob[i] > maxprob[best]) best = i;
      sel.push_back(best);
    }
  } else {
    std::vector<int> order = unc;
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return maxprob[a] > maxprob[b]; });
    int take = std::min<int>(k, int(order.size()));
    sel.assign(order.begin(), order.begin() + take);
  }
  for (int i : sel) { tokens[i] = argmax[i]; committed[i] = 1; }
  return int(sel.size());
}

}  // extern "C"

namespace {

// One forward pass of n tokens at positions pos0.. over the KV cache.
//  tokens[n], s[n][d] (nullptr = zeros), causal attention (prefill) or block-bidirectional.
//  Writes K/V rows [pos0, pos0+n) of every layer.  If xf != nullptr it receives the
//  final normalised hidden state [n][d] (the LM head input).
void forward(const orc_model& M, const orc_cfg& C, const int* tokens, const double* s, int n,
             int pos0, bool causal, orc_kv& kv, double* xf, double* qm = nullptr) {
  const int d = C.d, Hq = C.n_q_heads, Hkv = C.n_kv_heads, hd = C.head_dim, F = C.ffn;
  const bool rnd = C.act_round != 0, fp4 = C.act_fp4 != 0;
  const int nqkv = (Hq + 2 * Hkv) * hd;
  std::vector<double> h(size_t(n) * d), tmp(size_t(n) * d), xn(size_t(n) * d);
  // embedding + residual self-conditioning (R1, R2)
  for (int i = 0; i < n; ++i) mat_row(M.embed, tokens[i], h.data() + size_t(i) * d);
  if (s) {
    linear(s, n, M.w_adapter, tmp.data(), false);
    for (size_t i = 0; i < h.size(); ++i) h[i] += tmp[i];
  }
  std::vector<double> qkv(size_t(n) * nqkv), q(size_t(n) * Hq * hd), o(size_t(n) * Hq * hd);
  std::vector<double> g(size_t(n) * F), u(size_t(n) * F), a(size_t(n) * F);
  for (int l = 0; l < C.n_layers; ++l) {
    const orc_layer& L = M.layers[l];
    double* kl = kv.k + size_t(l) * Hkv * kv.max_ctx * hd;
    double* vl = kv.v + size_t(l) * Hkv * kv.max_ctx * hd;
    // attention sub-block
    for (int i = 0; i < n; ++i) rmsnorm(h.data() + size_t(i) * d, d, L.attn_norm, C.rms_eps, xn.data() + size_t(i) * d);
    linear(xn.data(), n, L.w_qkv, qkv.data(), fp4, qm);
    for (int i = 0; i < n; ++i) {
      double* row = qkv.data() + size_t(i) * nqkv;
      long pos = pos0 + i;
      for (int hh = 0; hh < Hq + Hkv; ++hh) rope(row + hh * hd, hd, pos, C.rope_theta);
      const bool fp8 = C.kv_fp8 != 0;
      for (int e = 0; e < nqkv; ++e)
        if (!(fp8 && e >= Hq * hd)) row[e] = maybe_round(row[e], rnd);  // K/V rows: see R13 below
      if (fp8)
        for (int hh = Hq; hh < Hq + 2 * Hkv; ++hh) orc_kv_quantize_row(row + hh * hd, hd, nullptr, row + hh * hd);
      for (int hh = 0; hh < Hq; ++hh)
        std::memcpy(q.data() + (size_t(i) * Hq + hh) * hd, row + hh * hd, hd * sizeof(double));
      for (int gg = 0; gg < Hkv; ++gg) {
        std::memcpy(kl + (size_t(gg) * kv.max_ctx + pos) * hd, row + (Hq + gg) * hd, hd * sizeof(double));
        std::memcpy(vl + (size_t(gg) * kv.max_ctx + pos) * hd, row + (Hq + Hkv + gg) * hd, hd * sizeof(double));
      }
    }
    orc_attention(q.data(), n, Hq, Hkv, hd, kl, vl, kv.max_ctx, pos0, causal ? 1 : 0, o.data());
    linear(o.data(), n, L.w_o, tmp.data(), fp4, qm);
    for (size_t i = 0; i < h.size(); ++i) h[i] += tmp[i];
    // MLP sub-block
    for (int i = 0; i < n; ++i) rmsnorm(h.data() + size_t(i) * d, d, L.mlp_norm, C.rms_eps, xn.data() + size_t(i) * d);
    linear(xn.data(), n, L.w_gate, g.data(), fp4, qm);
    linear(xn.data(), n, L.w_up, u.data(), fp4, qm);
    for (size_t i = 0; i < a.size(); ++i) {
      double silu = g[i] / (1.0 + std::exp(-g[i]));
      a[i] = silu * u[i];
    }
    linear(a.data(), n, L.w_down, tmp.data(), fp4, qm);
    for (size_t i = 0; i < h.size(); ++i) h[i] += tmp[i];
  }
  if (xf) {
    for (int i = 0; i < n; ++i) rmsnorm(h.data() + size_t(i) * d, d, M.final_norm, C.rms_eps, xf + size_t(i) * d);
  }
}

}  // namespace

extern "C" {

// Block state of one denoising block (R2): tokens (MASK or committed id), committed flags,
// residual input s (zero rows where there is no residual), and the round counter.
typedef struct orc_block {
  int* tokens;        // [B]
  uint8_t* committed; // [B]
  double* s;          // [B][d]
  int round;
} orc_block;

void orc_forward(const orc_model* M, const orc_cfg* C, const int* tokens, const double* s, int n,
                 int pos0, int causal, orc_kv* kv, double* xf) {
  forward(*M, *C, tokens, s, n, pos0, causal != 0, *kv, xf);
}

// One denoising round at prefix length L ([blog] "What shipped"; [card] SDAR flags).
// Outputs the row statistics of the round (st[B]) and updates the block state in place.
// Returns the number of positions committed.
int orc_round(const orc_model* M, const orc_cfg* C, orc_block* blk, orc_kv* kv, int L, double tau,
              int mode, int k, orc_stats* st) {
  const int B = C->block_size, d = C->d;
  std::vector<double> xf(size_t(B) * d), snext(size_t(B) * d), qm(B, std::numeric_limits<double>::infinity());
  forward(*M, *C, blk->tokens, blk->s, B, L, false, *kv, xf.data(), qm.data());
  orc_lmhead(xf.data(), B, &M->embed, C->mask_id, C->act_fp4, nullptr, st, snext.data(), nullptr);
  for (int i = 0; i < B; ++i) st[i].qmargin = std::min(st[i].qmargin, qm[i]);
  std::vector<double> mp(B);
  std::vector<int> am(B);
  for (int i = 0; i < B; ++i) { mp[i] = st[i].maxprob; am[i] = st[i].argmax; }
  int nc = orc_commit(B, mp.data(), am.data(), tau, mode, k, blk->tokens, blk->committed);
  for (int i = 0; i < B; ++i)
    for (int c = 0; c < d; ++c)
      blk->s[size_t(i) * d + c] = blk->committed[i] ? 0.0 : snext[size_t(i) * d + c];
  blk->round += 1;
  return nc;
}

// Decode one block at prefix length L: rounds until every position is committed (or the
// round cap B is reached), then the clean KV-fill forward (R5).  Returns the number of
// rounds, or -1 if the cap was hit with positions still uncommitted.
int orc_decode_block(const orc_model* M, const orc_cfg* C, orc_kv* kv, int L, double tau, int mode,
                     int k, int* tokens_out) {
  const int B = C->block_size, d = C->d;
  std::vector<int> tokens(B, C->mask_id);
  std::vector<uint8_t> committed(B, 0);
  std::vector<double> s(size_t(B) * d, 0.0);
  std::vector<orc_stats> st(B);
  orc_block blk{tokens.data(), committed.data(), s.data(), 0};
  auto any_unc = [&] { for (int i = 0; i < B; ++i) if (!committed[i]) return true; return false; };
  while (any_unc() && blk.round < B) orc_round(M, C, &blk, kv, L, tau, mode, k, st.data());
  if (any_unc()) return -1;
  forward(*M, *C, tokens.data(), nullptr, B, L, false, *kv, nullptr);
  std::memcpy(tokens_out, tokens.data(), B * sizeof(int));
  return blk.round;
}

void orc_prefill(const orc_model* M, const orc_cfg* C, orc_kv* kv, const int* prompt, int P) {
  forward(*M, *C, prompt, nullptr, P, 0, true, *kv, nullptr);
}

// Prefill + blocks until max_new tokens (rounded up to whole blocks, then truncated).
// Returns the number of blocks, or -1 on a round-cap failure.
int orc_generate(const orc_model* M, const orc_cfg* C, orc_kv* kv, const int* prompt, int P,
                 int max_new, double tau, int mode, int k, int* out, int* rounds_per_block) {
  const int B = C->block_size;
  orc_prefill(M, C, kv, prompt, P);
  int nblk = (max_new + B - 1) / B;
  std::vector<int> blk(B);
  for (int b = 0; b < nblk; ++b) {
    int r = orc_decode_block(M, C, kv, P + b * B, tau, mode, k, blk.data());
    if (r < 0) return -1;
    rounds_per_block[b] = r;
    for (int i = 0; i < B && b * B + i < max_new; ++i) out[b * B + i] = blk[i];
  }
  return nblk;
}

}  // extern "C"

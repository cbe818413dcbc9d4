// dlm_ops.cu -- the light kernels of a denoising round: they consume the GEMM partial
// sums and apply what follows each projection, plus the LM-head statistics and the
// commit rule.
//
// Round data flow (one block of T = B tokens at positions L .. L+B-1):
//   s (fp32) --bf16--> W_a GEMM --k_embed_adapter_norm--> h = E[x] + W_a s, xn = RMSNorm(h)
//   per layer: QKV GEMM --k_qkv_rope--> q, K/V cache rows [L, L+B) (RoPE, bf16)
//              attention --> o (bf16)
//              O GEMM --k_residual_norm--> h += o W_o^T, xn = RMSNorm(h)
//              gate/up GEMM --k_silu_gate--> a = silu(g) * u (bf16)
//              down GEMM --k_residual_norm--> h += a W_d^T, xn = RMSNorm(h) (next norm)
//   LM head: E GEMM --> logits --k_rowstats--> stats, P = softmax (bf16)
//            P E (MN-major GEMM) --k_store_rows--> s
//   k_commit: commit rule, loop condition.
#include <cfloat>
#include <cstdio>

#include "dlm_device.cuh"
#include "dlm_internal.h"
#include "dlm_ops.h"

namespace dlm {

// ------------------------------------------------------------------ block reductions
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nw = blockDim.x / 32;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < nw; ++i) r += red[i];  // fixed order: deterministic
  return r;
}

// ------------------------------------------------------------------ tile finishers
// The finishers sum a GEMM's per-slot partials ([tile][slot][TP][128], slot order) for one
// tile and 32 tokens (grid: tiles x ceil(T / 32)) and apply the op.  256 threads; a thread
// owns a pair of tile rows for 8 tokens, so RoPE (rows j, j + hd/2) and SiLU-mul (gate row
// r, up row r + 64) combine values the same thread loaded: no shared memory, no barrier.
// All loads of a thread are issued before any sum.
constexpr int kFinTok = 8;    // tokens per thread
constexpr int kFinSlots = 4;  // slots loaded per batch

// v[a|b][j] = sum over slots of rows ra / rb, tokens t0 + j (0 where t0 + j >= T)
__device__ __forceinline__ void finish_load_pair(const GemmOut& o, int tile, int ra, int rb, int t0,
                                                 float (&va)[kFinTok], float (&vb)[kFinTok]) {
  const int TP = (o.T + 31) / 32 * 32;
  const int ns = tile_slots(o, tile);
  const float* base = o.partial + (size_t)tile * o.max_slots * kTileM * TP + (size_t)t0 * kTileM;
#pragma unroll
  for (int j = 0; j < kFinTok; ++j) { va[j] = 0.f; vb[j] = 0.f; }
  for (int sl = 0; sl < ns; sl += kFinSlots) {
    float xa[kFinSlots][kFinTok], xb[kFinSlots][kFinTok];
#pragma unroll
    for (int b = 0; b < kFinSlots; ++b) {
      const float* p = base + (size_t)(sl + b) * kTileM * TP;
      const bool ok = sl + b < ns;
#pragma unroll
      for (int j = 0; j < kFinTok; ++j) {
        const bool in = ok && t0 + j < o.T;
        xa[b][j] = in ? __ldcg(p + (size_t)j * kTileM + ra) : 0.f;
        xb[b][j] = in ? __ldcg(p + (size_t)j * kTileM + rb) : 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < kFinSlots; ++b)
#pragma unroll
      for (int j = 0; j < kFinTok; ++j) { va[j] += xa[b][j]; vb[j] += xb[b][j]; }
  }
}

// QKV: RoPE (NeoX pairs j, j + hd/2, angles from the fp64-built table) on q and k heads;
// q as bf16 [T][Hq][hd], K and V rows into the cache at positions L + t: bf16, or for an FP8
// cache e4m3 codes with one fp32 scale amax / 448 per (KV head, position) row.  A thread owns
// the pair (jj, jj + hd/2) of one head for 8 tokens; the pairs of one head row are held by
// min(32, hd/2) consecutive lanes, and by two warps for hd = 128 (their maxima meet in shared
// memory).
__global__ void __launch_bounds__(256) k_finish_qkv(FinishArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float amax2[4][kFinTok][2];  // [token group][token][warp of the pair] (hd = 128)
  const EpiArgs& e = a.epi;
  const bool fp8 = e.kc8 != nullptr;
  const int tile = blockIdx.x, p = threadIdx.x % 64, tg = threadIdx.x / 64;
  const int t0 = blockIdx.y * 32 + tg * kFinTok;
  const int half = e.hd / 2;
  const int ra = (p / half) * e.hd + p % half, rb = ra + half;  // rows of the pair in the tile
  const int n = tile * kTileM + ra;                              // feature of row ra
  const bool active = n < a.N && t0 < a.out.T;
  if (!active && !fp8) return;  // (the FP8 path reduces across threads: no early exit)
  const int L = e.pos0_dev ? *e.pos0_dev + e.pos_off : e.pos0;
  float va[kFinTok], vb[kFinTok];
  if (active) {
    finish_load_pair(a.out, tile, ra, rb, t0, va, vb);
  } else {
#pragma unroll
    for (int j = 0; j < kFinTok; ++j) va[j] = vb[j] = 0.f;
  }
  const int hh = n / e.hd, jj = n % e.hd;  // jj < half
  const bool rope = hh < e.Hq + e.Hkv;
  float x0[kFinTok], x1[kFinTok];
#pragma unroll
  for (int j = 0; j < kFinTok; ++j) {
    const bool in = active && t0 + j < a.out.T;
    const float2 cs = (rope && in) ? e.rope_tab[(size_t)(L + t0 + j) * half + jj] : make_float2(1.f, 0.f);
    x0[j] = va[j] * cs.x - vb[j] * cs.y;
    x1[j] = va[j] * cs.y + vb[j] * cs.x;
  }
  if (active && hh < e.Hq) {
    __nv_bfloat16* dst = e.q + (size_t)t0 * e.Hq * e.hd + (size_t)hh * e.hd + jj;
    const size_t stride_t = (size_t)e.Hq * e.hd;
#pragma unroll
    for (int j = 0; j < kFinTok; ++j) {
      if (t0 + j < a.out.T) {
        dst[(size_t)j * stride_t] = f2bf(x0[j]);
        dst[(size_t)j * stride_t + half] = f2bf(x1[j]);
      }
    }
  }
  const bool is_k = hh >= e.Hq && hh < e.Hq + e.Hkv;
  const int kvh = is_k ? hh - e.Hq : hh - e.Hq - e.Hkv;  // KV head of a K or V row
  if (!fp8) {
    if (!active || hh < e.Hq) return;
    __nv_bfloat16* dst = (is_k ? e.kc : e.vc) + ((size_t)kvh * e.max_ctx + L + t0) * e.hd + jj;
#pragma unroll
    for (int j = 0; j < kFinTok; ++j) {
      if (t0 + j < a.out.T) {
        dst[(size_t)j * e.hd] = f2bf(x0[j]);
        dst[(size_t)j * e.hd + half] = f2bf(x1[j]);
      }
    }
    return;
  }
  // FP8: row amax over the head's pairs (every thread takes part; inactive ones carry 0)
  const int lane = threadIdx.x % 32;
  const int group = half < 32 ? half : 32;  // lanes of one head row within a warp
  float am[kFinTok];
#pragma unroll
  for (int j = 0; j < kFinTok; ++j) {
    float v = fmaxf(fabsf(x0[j]), fabsf(x1[j]));
    for (int o = group / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    am[j] = v;
  }
  if (half == 64) {  // the row spans the two warps of this token group
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < kFinTok; ++j) amax2[tg][j][(threadIdx.x / 32) % 2] = am[j];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kFinTok; ++j) am[j] = fmaxf(amax2[tg][j][0], amax2[tg][j][1]);
  }
  if (!active || hh < e.Hq) return;
  uint8_t* dst = (is_k ? e.kc8 : e.vc8) + ((size_t)kvh * e.max_ctx + L + t0) * e.hd + jj;
  float* sdst = (is_k ? e.ks : e.vs) + (size_t)kvh * e.max_ctx + L + t0;
#pragma unroll
  for (int j = 0; j < kFinTok; ++j) {
    if (t0 + j >= a.out.T) continue;
    const float sc = am[j] / 448.0f;
    uint8_t c0 = 0, c1 = 0;
    if (sc > 0.f) {
      const float r0 = x0[j] / sc, r1 = x1[j] / sc;
      c0 = (uint8_t)(e4m3_rne_bits(fabsf(r0)) | (r0 < 0.f ? 0x80 : 0));
      c1 = (uint8_t)(e4m3_rne_bits(fabsf(r1)) | (r1 < 0.f ? 0x80 : 0));
    }
    dst[(size_t)j * e.hd] = c0;
    dst[(size_t)j * e.hd + half] = c1;
    if (jj == 0) sdst[j] = sc;
  }
}

// gate/up pair tile (gate features in rows 0..63, up in 64..127): act = silu(g) u as a split
// bf16 pair.  With act_amax set (the down projection is NVFP4) the tile also leaves, per
// token, the largest magnitude of the values it stored (hi + lo), the partial maxima the
// wide quantizer takes the row scale from.
__global__ void __launch_bounds__(256) k_finish_silu(FinishArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float am2[4][kFinTok][2];
  const EpiArgs& e = a.epi;
  const int tile = blockIdx.x, r = threadIdx.x % 64, tg = threadIdx.x / 64;
  const int t0 = blockIdx.y * 32 + tg * kFinTok;
  const int f = tile * 64 + r;
  const bool active = f < a.N && t0 < a.out.T;
  if (!active && !e.act_amax) return;
  float g[kFinTok], u[kFinTok], am[kFinTok];
  if (active) finish_load_pair(a.out, tile, r, r + 64, t0, g, u);
#pragma unroll
  for (int j = 0; j < kFinTok; ++j) {
    am[j] = 0.f;
    if (active && t0 + j < a.out.T) {
      float v = g[j] / (1.0f + expf(-g[j])) * u[j];
      if (e.route_w) v *= e.route_w[(size_t)(t0 + j) * e.route_e + f / e.route_f];
      __nv_bfloat16* p = e.act + (size_t)(t0 + j) * a.N + f;
      store_split(p, e.act_lo, v);
      if (e.act_amax) {
        const __nv_bfloat16 h = f2bf(v);
        am[j] = fabsf(bf2f(h) + bf2f(f2bf(v - bf2f(h))));  // the value the quantizer reads
      }
    }
  }
  if (!e.act_amax) return;
  // tile maximum per token: 64 features = the two warps of this token group
#pragma unroll
  for (int j = 0; j < kFinTok; ++j) am[j] = warp_max(am[j]);
  if (threadIdx.x % 32 == 0)
#pragma unroll
    for (int j = 0; j < kFinTok; ++j) am2[tg][j][(threadIdx.x / 32) % 2] = am[j];
  __syncthreads();
  if (threadIdx.x % 64 == 0)
#pragma unroll
    for (int j = 0; j < kFinTok; ++j)
      if (t0 + j < a.out.T) e.act_amax[(size_t)tile * a.out.T + t0 + j] = fmaxf(am2[tg][j][0], am2[tg][j][1]);
}

// Routed-expert MLP front, in two kernels.
// k_moe_logits, grid (T, ceil(E / 8)): CTA (t, c) normalises row t, x = h / sqrt(mean(h^2) + eps)
// g (fp32; CTA (t, 0) also stores it), and its 8 warps take the router logits of experts
// 8 c .. 8 c + 7, l_e = x . W_r[e] (W_r bf16, fp32 sums).
__global__ void __launch_bounds__(256) k_moe_logits(MoeRouteArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float sx[];  // x [d]
  __shared__ float red[8];
  const int t = blockIdx.x, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const float* h = a.h + (size_t)t * a.d;
  float ss = 0.f;
  for (int c = tid; c < a.d; c += 256) ss += h[c] * h[c];
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += red[w];
  const float r = 1.0f / sqrtf(tot / (float)a.d + a.eps);
  for (int c = tid; c < a.d; c += 256) {
    const float xv = h[c] * r * bf2f(a.g[c]);
    sx[c] = xv;
    if (blockIdx.y == 0) a.x[(size_t)t * a.d + c] = xv;
  }
  __syncthreads();
  const int e = blockIdx.y * 8 + warp;
  if (e >= a.E) return;
  const __nv_bfloat16* wr = a.wr + (size_t)e * a.d;
  float acc = 0.f;
  for (int c0 = lane * 8; c0 < a.d; c0 += 256) {
    const uint4 raw = *reinterpret_cast<const uint4*>(wr + c0);
    const __nv_bfloat16* wv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += sx[c0 + u] * bf2f(wv[u]);
  }
  acc = warp_sum(acc);
  if (lane == 0) a.logits[(size_t)t * a.E + e] = acc;
}

// k_moe_topk, one warp per row: the k largest logits (ties to the lower index), weighted by
// softmax renormalised over the chosen, w_e = exp(l_e - m) / sum_chosen exp(l_j - m); route_w
// gets the weights densely (zero for the experts not chosen).
__global__ void __launch_bounds__(256) k_moe_topk(MoeRouteArgs a) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (t >= a.T) return;
  const float* l = a.logits + (size_t)t * a.E;
  float lv[8];  // lane owns experts lane + 32 j (E <= 256)
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    lv[j] = e < a.E ? l[e] : -INFINITY;
    mx = fmaxf(mx, lv[j]);
  }
  mx = warp_max(mx);
  uint32_t taken = 0;
  float zs = 0.f, pw[8];
  int pi[8];
  for (int s = 0; s < a.k; ++s) {
    float best = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (e < a.E && !((taken >> j) & 1u) && (lv[j] > best || (lv[j] == best && e < be))) { best = lv[j]; be = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float b2 = __shfl_xor_sync(0xffffffffu, best, o);
      const int e2 = __shfl_xor_sync(0xffffffffu, be, o);
      if (b2 > best || (b2 == best && e2 < be)) { best = b2; be = e2; }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    pi[s] = be;
    pw[s] = expf(best - mx);
    zs += pw[s];
  }
  for (int e = lane; e < a.E; e += 32) a.route_w[(size_t)t * a.E + e] = 0.f;
  __syncwarp();
  if (lane == 0)
    for (int s = 0; s < a.k; ++s) {
      const float w = pw[s] / zs;
      a.route_w[(size_t)t * a.E + pi[s]] = w;
      if (a.topk_idx) a.topk_idx[(size_t)t * a.k + s] = pi[s];
      if (a.topk_w) a.topk_w[(size_t)t * a.k + s] = w;
    }
}

// out[t][n] = scale * y (scale 0 means 1) (+ add[t][n]): one thread per feature n of the tile
// and token t (grid: tiles x T, 128 threads), its slots summed in slot order, eight loads in
// flight.
__global__ void __launch_bounds__(128) k_finish_store(FinishArgs a) {
  pdl_trigger();
  pdl_wait();
  const EpiArgs& e = a.epi;
  const GemmOut& o = a.out;
  const int tile = blockIdx.x, t = blockIdx.y, row = threadIdx.x;
  const int n = tile * kTileM + row;
  if (t >= o.T || n >= a.N) return;
  const size_t TP = (size_t)(o.T + 31) / 32 * 32, ss = TP * kTileM;
  const int ns = tile_slots(o, tile);
  const float* p = o.partial + ((size_t)tile * o.max_slots * TP + t) * kTileM + row;
  float v = 0.f;
  int sl = 0;
  for (; sl + 8 <= ns; sl += 8) {
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = __ldcg(p + (size_t)(sl + u) * ss);
#pragma unroll
    for (int u = 0; u < 8; ++u) v += x[u];
  }
  for (; sl < ns; ++sl) v += __ldcg(p + (size_t)sl * ss);
  const size_t i = (size_t)t * e.ld + n;
  e.out[i] = ((e.scale != 0.f) ? v * e.scale : v) + (e.add ? e.add[i] : 0.f);
}

// Residual update and RMSNorm of one token row, spread over a cluster of kRnCluster CTAs:
//   h[t] = h[t] + y[t]        (residual of a projection whose partial sums are in `out`)
//   h[t] = E[tok_t] + y[t]    (embedding, with y = W_a s, or y = 0 when out.partial is null)
//   xn[t] = h[t] / sqrt(mean(h[t]^2) + eps) * g   as a split bf16 pair.
// CTA rank r of token t's cluster owns features [r d/4, (r + 1) d/4); each of its 256
// threads owns features r d/4 + threadIdx.x + k 256 (k < kFeat) and issues the loads of all
// their slots (up to kSlotsReg each) before summing them in slot order.  The four partial
// sums of squares are exchanged through distributed shared memory and added in rank order.
constexpr int kRnThreads = 256;
constexpr int kFeat = 4;
constexpr int kSlotsReg = 12;
__global__ void __launch_bounds__(kRnThreads) k_resid_norm(ResNormArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[kRnThreads / 32];
  __shared__ float ss_all[kRnCluster], amax_all[kRnCluster];
  __shared__ int nsl[16];
  const int t = blockIdx.x / kRnCluster;
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const int dq = a.d / kRnCluster, f0 = (int)rank * dq;
  const GemmOut& o = a.out;
  const bool has_y = o.partial != nullptr;
  const uint32_t TP = (uint32_t)(o.T + 31) / 32 * 32;
  const uint32_t st = TP * kTileM;
  const int tile0 = f0 >> 7, ntl = ((f0 + dq - 1) >> 7) - tile0 + 1;  // tiles of this CTA's features
  if (has_y && (int)threadIdx.x < ntl) nsl[threadIdx.x] = tile_slots(o, tile0 + threadIdx.x);
  __syncthreads();
  const bool emb = a.embed || a.embed_codes;
  const int tok = !emb ? 0 : ((a.tokens2 && t >= a.tok_split) ? a.tokens2[t - a.tok_split] : a.tokens[t]);
  float base[kFeat], x[kFeat][kSlotsReg];
  int ns[kFeat];
  const float* pp[kFeat];
#pragma unroll
  for (int k = 0; k < kFeat; ++k) {
    const int n = f0 + threadIdx.x + k * kRnThreads;
    const bool ok = (int)threadIdx.x + k * kRnThreads < dq;
    ns[k] = (ok && has_y) ? nsl[(n >> 7) - tile0] : 0;
    pp[k] = has_y ? o.partial + ((size_t)(n >> 7) * o.max_slots * TP + t) * kTileM + (n & 127) : nullptr;
    if (!ok) {
      base[k] = 0.f;
    } else if (a.embed_codes) {  // NVFP4 E: code x e4m3 scale (exact in fp32), times the tensor scale
      const uint8_t cb = a.embed_codes[(size_t)tok * (a.d / 2) + n / 2];
      base[k] = e2m1_value_dev((n & 1) ? (uint8_t)(cb >> 4) : (uint8_t)(cb & 15)) *
                e4m3_value_dev(a.embed_sc[(size_t)tok * (a.d / 16) + n / 16]) * a.embed_scale;
    } else {
      base[k] = a.embed ? bf2f(a.embed[(size_t)tok * a.d + n]) * a.embed_scale : a.h[(size_t)t * a.d + n];
    }
#pragma unroll
    for (int sl = 0; sl < kSlotsReg; ++sl) x[k][sl] = sl < ns[k] ? __ldcg(pp[k] + sl * st) : 0.f;
  }
  float hv[kFeat];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kFeat; ++k) {
    float y = 0.f;
#pragma unroll
    for (int sl = 0; sl < kSlotsReg; ++sl) y += x[k][sl];  // slot order
    for (int sl = kSlotsReg; sl < ns[k]; ++sl) y += __ldcg(pp[k] + sl * st);
    hv[k] = base[k] + y;
    const int n = f0 + threadIdx.x + k * kRnThreads;
    if ((int)threadIdx.x + k * kRnThreads < dq) {
      a.h[(size_t)t * a.d + n] = hv[k];
      ss += hv[k] * hv[k];
    }
  }
  ss = block_sum(ss, red);
  if (threadIdx.x < kRnCluster) {
    // this CTA's partial into slot `rank` of every CTA of the cluster (itself included)
    uint32_t dst;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(dst) : "r"(smem_u32(&ss_all[rank])), "r"((uint32_t)threadIdx.x));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst), "f"(ss) : "memory");
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  float tot = 0.f;
#pragma unroll
  for (int q = 0; q < kRnCluster; ++q) tot += ss_all[q];  // rank order: the same sum everywhere
  const float r = 1.0f / sqrtf(tot / (float)a.d + a.eps);
  float xv[kFeat];
#pragma unroll
  for (int k = 0; k < kFeat; ++k) {
    const int n = f0 + threadIdx.x + k * kRnThreads;
    xv[k] = 0.f;
    if ((int)threadIdx.x + k * kRnThreads < dq) {
      xv[k] = hv[k] * r * bf2f(a.gain[n]);
      store_split(a.xn + (size_t)t * a.d + n, a.xn_lo, xv[k]);
    }
  }
  if (a.qcodes == nullptr) return;
  // NVFP4 input of the next GEMM (the quantizer of k_act_quant on the fp32 row): row scale
  // from the amax over the cluster, then 16-element groups = half-warps (the features of a
  // warp for one k are 32 consecutive ones; d / 4 is a multiple of 64 here)
  float am = 0.f;
#pragma unroll
  for (int k = 0; k < kFeat; ++k) am = fmaxf(am, fabsf(xv[k]));
  am = warp_max(am);
  __syncthreads();  // red[] is reused
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = am;
  __syncthreads();
  if (threadIdx.x < kRnCluster) {
    float m = 0.f;
    for (int i = 0; i < kRnThreads / 32; ++i) m = fmaxf(m, red[i]);
    uint32_t dst;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(dst) : "r"(smem_u32(&amax_all[rank])), "r"((uint32_t)threadIdx.x));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst), "f"(m) : "memory");
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  float amax = 0.f;
#pragma unroll
  for (int q = 0; q < kRnCluster; ++q) amax = fmaxf(amax, amax_all[q]);
  const float S = amax / (6.0f * 448.0f);
  if (rank == 0 && threadIdx.x == 0) a.qsx[t] = S;
  const int lane = threadIdx.x % 32;
#pragma unroll
  for (int k = 0; k < kFeat; ++k) {
    if ((int)(threadIdx.x - lane) + k * kRnThreads >= dq) continue;  // whole warp out of range
    const int n = f0 + threadIdx.x + k * kRnThreads;
    float bm = fabsf(xv[k]);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));  // within the half-warp
    const uint8_t sb = (S > 0.f) ? e4m3_rne_bits(bm / (6.0f * S)) : 0;
    const float denom = e4m3_value_dev(sb) * S;
    const uint32_t code = denom > 0.f ? e2m1_rne(xv[k] / denom) : 0u;
    const uint32_t hi = __shfl_down_sync(0xffffffffu, code, 1);
    if ((lane & 1) == 0) a.qcodes[(size_t)t * (a.d / 2) + n / 2] = (uint8_t)(code | (hi << 4));
    if ((lane & 15) == 0) {
      const int gi = n / 16;
      a.qscales[tok_scale_index(t, gi, a.d)] = sb;
    }
  }
}

// Split bf16 copy of s (the W_a GEMM input): high halves at y[i], low halves at y[i + lo];
// the first zero_n elements of y are zero (rows without a residual input), x fills the n
// after them.
__global__ void k_to_bf16(const float* x, __nv_bfloat16* y, long n, long lo, long zero_n) {
  pdl_trigger();
  pdl_wait();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < zero_n) store_split(y + i, lo, 0.f);
  else if (i < zero_n + n) store_split(y + i, lo, x[i - zero_n]);
}

// Row statistics, phase 1: for logits[b][chunk] (mask id excluded) the chunk's max m_c,
// its lowest argmax, Z_c = sum e^(l - m_c) and A_c = sum e^(l - m_c) (l - m_c).
// grid (n_chunks, B), 256 threads.
__global__ void k_rowstats_part(RowStatsArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red_v[32];
  __shared__ int red_i[32];
  __shared__ float bc;
  const int ch = blockIdx.x, b = blockIdx.y;
  const int v0 = ch * a.chunk, v1 = min(a.V, v0 + a.chunk);
  const float* l = a.logits + (size_t)b * a.ld;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nw = blockDim.x / 32;
  float m = -INFINITY;
  int am = 0x7fffffff;
  for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
    if (v == a.mask_id) continue;
    const float x = l[v];
    if (x > m || (x == m && v < am)) { m = x; am = v; }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const int a2 = __shfl_xor_sync(0xffffffffu, am, o);
    if (m2 > m || (m2 == m && a2 < am)) { m = m2; am = a2; }
  }
  if (lane == 0) { red_v[warp] = m; red_i[warp] = am; }
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = red_v[0];
    int aa = red_i[0];
    for (int i = 1; i < nw; ++i)
      if (red_v[i] > mm || (red_v[i] == mm && red_i[i] < aa)) { mm = red_v[i]; aa = red_i[i]; }
    bc = mm;
    red_i[0] = aa;
  }
  __syncthreads();
  m = bc;
  am = red_i[0];
  __syncthreads();
  float z = 0.f, A = 0.f;
  if (m > -INFINITY) {
    for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
      if (v == a.mask_id) continue;
      const float x = l[v] - m;
      const float ex = expf(x);
      z += ex;
      A += ex * x;
    }
  }
  z = block_sum(z, red_v);
  A = block_sum(A, red_v);
  if (threadIdx.x == 0) {
    float4* p = reinterpret_cast<float4*>(a.part) + (size_t)b * gridDim.x + ch;
    *p = make_float4(m, __int_as_float(am), z, A);
  }
}

// Row statistics, phase 2: merges the chunk partials of row b (every CTA redundantly, in
// chunk order), chunk 0 writes the statistics, and every CTA writes its chunk of
// P = softmax as a split bf16 pair.  Merge: M = max m_c, Z = sum_c e^(m_c - M) Z_c,
// A = sum_c e^(m_c - M) (A_c + (m_c - M) Z_c); lse = M + ln Z, maxprob = 1/Z,
// entropy = ln Z - A / Z.  grid (n_chunks, B), 256 threads.
__global__ void k_rowstats_final(RowStatsArgs a) {
  pdl_trigger();
  pdl_wait();
  const int ch = blockIdx.x, b = blockIdx.y, nch = gridDim.x;
  const float4* part = reinterpret_cast<const float4*>(a.part) + (size_t)b * nch;
  float M = -INFINITY;
  int am = 0x7fffffff;
  for (int i = 0; i < nch; ++i) {
    const float4 q = part[i];
    const int ai = __float_as_int(q.y);
    if (q.x > M) { M = q.x; am = ai; }  // chunks in id order: the first maximal chunk wins
  }
  float Z = 0.f, A = 0.f;
  for (int i = 0; i < nch; ++i) {
    const float4 q = part[i];
    if (q.x == -INFINITY) continue;
    const float w = expf(q.x - M);
    Z += w * q.z;
    A += w * (q.w + (q.x - M) * q.z);
  }
  const float lnz = logf(Z);
  const float lse = M + lnz;
  if (ch == 0 && threadIdx.x == 0) {
    a.stats.m[b] = M;
    a.stats.lse[b] = lse;
    a.stats.maxprob[b] = 1.0f / Z;
    a.stats.entropy[b] = lnz - A / Z;
    a.stats.argmax[b] = am;
  }
  if (a.P) {
    const int v0 = ch * a.chunk, v1 = min(a.V, v0 + a.chunk);
    const float* l = a.logits + (size_t)b * a.ld;
    __nv_bfloat16* p = a.P + (size_t)b * a.V;
    for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x)
      store_split(p + v, a.P_lo, v == a.mask_id ? 0.f : expf(l[v] - lse));
  }
}

// Commit rule for one block (one CTA of kCommitThreads >= B threads).  Threshold mode: every uncommitted
// position with maxprob >= tau, or if none qualifies the single uncommitted position with
// the largest maxprob (ties -> lowest position).  Top-k mode: the min(k, remaining)
// uncommitted positions of largest maxprob (ties -> lowest position).  Newly committed
// positions take their argmax token and get a zero residual row.
__global__ void k_commit(CommitArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float mp[64];
  __shared__ int unc[64];
  __shared__ int sel[64];
  __shared__ int best;
  const int i = threadIdx.x;
  const int B = a.B;
  if (i < B) {
    mp[i] = a.maxprob[i];
    unc[i] = a.committed[i] ? 0 : 1;
    sel[i] = 0;
  }
  __syncthreads();
  if (a.mode == DLM_COMMIT_THRESHOLD) {
    int q = (i < B && unc[i] && mp[i] >= a.tau) ? 1 : 0;
    if (i < B) sel[i] = q;
    int nq = __syncthreads_count(q);
    if (nq == 0 && i == 0) {
      int bi = -1;
      for (int j = 0; j < B; ++j)
        if (unc[j] && (bi < 0 || mp[j] > mp[bi])) bi = j;
      best = bi;
    }
    __syncthreads();
    if (nq == 0 && i < B) sel[i] = (i == best) ? 1 : 0;
  } else {
    if (i < B && unc[i]) {
      int rank = 0;
      for (int j = 0; j < B; ++j)
        if (unc[j] && (mp[j] > mp[i] || (mp[j] == mp[i] && j < i))) ++rank;
      sel[i] = rank < a.k ? 1 : 0;
    }
  }
  __syncthreads();
  if (i < B && sel[i]) {
    a.tokens[i] = a.argmax[i];
    a.committed[i] = 1;
  }
  __syncthreads();
  // committed positions (old and new) carry no residual into the next round: every thread
  // zeroes a strided share of those rows (float4 stores when s is 16-byte aligned)
  if (((uintptr_t)a.s & 15) == 0 && (a.d & 3) == 0) {
    const int d4 = a.d / 4;
    float4* s4 = reinterpret_cast<float4*>(a.s);
    for (int e = threadIdx.x; e < B * d4; e += blockDim.x) {
      const int r = e / d4;
      if (!unc[r] || sel[r]) s4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else {
    for (int e = threadIdx.x; e < B * a.d; e += blockDim.x) {
      const int r = e / a.d;
      if (!unc[r] || sel[r]) a.s[e] = 0.f;
    }
  }
  int left = (i < B && unc[i] && !sel[i]) ? 1 : 0;
  int nleft = __syncthreads_count(left);
  if (i == 0) {
    int rnd = *a.round + 1;
    *a.round = rnd;
    unsigned cond = (nleft > 0 && rnd < B) ? 1u : 0u;
    if (nleft > 0 && rnd >= B && a.status) atomicCAS(a.status, 0, DLM_EROUNDCAP);
    if (a.use_cond) cudaGraphSetConditional(a.cond, cond);
  }
}

// tokens = mask_id, committed = 0, s = 0, round = 0, status = 0.
__global__ void k_block_init(BlockInitArgs a) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < a.B) {
    a.tokens[i] = a.mask_id;
    a.committed[i] = 0;
  }
  if (i == 0) {
    *a.round = 0;
    if (a.status) *a.status = 0;
  }
  for (long n = i; n < (long)a.B * a.d; n += (long)gridDim.x * blockDim.x) a.s[n] = 0.f;
}

// End of a block: copy tokens and {round, status} out (and keep the tokens for the block's
// deferred KV-fill), merge the kernel error flag into the status, and advance the device
// prefix length by B.
__global__ void k_block_finish(BlockFinishArgs a) {
  pdl_trigger();
  pdl_wait();
  const int i = threadIdx.x;
  if (i < a.B) a.tokens_out[i] = a.tokens[i];
  if (i < a.B && a.pend_tokens) a.pend_tokens[i] = a.tokens[i];
  if (i == 0) {
    a.rounds_out[0] = *a.round;
    int st = *a.status;
    if (st == 0 && a.err) st = *a.err;
    a.rounds_out[1] = st;
    if (a.L_dev) *a.L_dev += a.B;
  }
}

__global__ void k_set_int(int* p, int v) {
  pdl_trigger();
  pdl_wait();
  *p = v;
}

// RoPE table: tab[p][j] = (cos, sin) of p * theta_j, theta_j = base^(-2j/hd), computed in
// double precision once per context (NeoX rotate-half pairing (j, j + hd/2)).
__global__ void k_rope_table(float2* tab, int max_ctx, int hd, double base) {
  const int half = hd / 2;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)max_ctx * half) return;
  const int p = (int)(i / half), j = (int)(i % half);
  const double theta = pow(base, -2.0 * (double)j / (double)hd);
  double s, c;
  sincos((double)p * theta, &s, &c);
  tab[i] = make_float2((float)c, (float)s);
}

// amax bits -> tensor scale amax / (6 * 448), in place.
__global__ void k_amax_to_scale(float* p) {
  pdl_trigger();
  pdl_wait();
  *p = __uint_as_float(*reinterpret_cast<unsigned*>(p)) / (6.0f * 448.0f);
}

// ------------------------------------------------------------------ NVFP4 quantizer
// Per-tensor scale S = amax / (6 * 448) (fp32 division), per 16-element block e4m3 scale
// sigma = RN_e4m3(amax_blk / (6 S)) (saturating), codes = RNE e2m1 of w / (sigma S).
__global__ void k_amax_bf16(const __nv_bfloat16* w, long n, unsigned* amax_bits) {
  pdl_trigger();
  pdl_wait();
  float m = 0.f;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(bf2f(w[i])));
  m = warp_max(m);
  if (threadIdx.x % 32 == 0) atomicMax(amax_bits, __float_as_uint(m));  // m >= 0: bit order = value order
}

__global__ void k_nvfp4_quantize(const __nv_bfloat16* w, int rows, int cols, uint8_t* codes,
                                 uint8_t* scales, const unsigned* amax_bits, float* tscale) {
  pdl_trigger();
  pdl_wait();
  const float amax = __uint_as_float(*amax_bits);
  const float S = amax / (6.0f * 448.0f);
  const long nblk = (long)rows * (cols / 16);
  const long b = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (b == 0 && tscale) *tscale = S;
  if (b >= nblk) return;
  const __nv_bfloat16* src = w + b * 16;
  float v[16];
  float bm = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) { v[j] = bf2f(src[j]); bm = fmaxf(bm, fabsf(v[j])); }
  uint8_t sb = (S > 0.f) ? e4m3_rne_bits(bm / (6.0f * S)) : 0;
  scales[b] = sb;
  const float denom = e4m3_value_dev(sb) * S;
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    uint8_t c0 = denom > 0.f ? e2m1_rne(v[j] / denom) : 0;
    uint8_t c1 = denom > 0.f ? e2m1_rne(v[j + 1] / denom) : 0;
    codes[b * 8 + j / 2] = (uint8_t)(c0 | (c1 << 4));
  }
}

// ------------------------------------------------------------------ NVFP4 activations
// One CTA (256 threads) per row; each thread owns up to kAqBlocks 16-element blocks.
constexpr int kAqBlocks = 4;
__global__ void __launch_bounds__(256) k_act_quant(ActQuantArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int t = blockIdx.x, nb = a.K / 16;
  float v[kAqBlocks][16];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kAqBlocks; ++i) {
    const int b = threadIdx.x + i * 256;
#pragma unroll
    for (int j = 0; j < 16; ++j) v[i][j] = 0.f;
    if (b < nb) {
      const size_t off = (size_t)t * a.K + (size_t)b * 16;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[i][j] = a.xf ? a.xf[off + j] : bf2f(a.xb[off + j]) + bf2f(a.xb[off + j + a.xb_lo]);
        amax = fmaxf(amax, fabsf(v[i][j]));
      }
    }
  }
  amax = warp_max(amax);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float m = threadIdx.x < 8 ? red[threadIdx.x] : 0.f;
    m = warp_max(m);
    if (threadIdx.x == 0) red[8] = m;
  }
  __syncthreads();
  const float S = red[8] / (6.0f * 448.0f);
  if (threadIdx.x == 0) a.sx[t] = S;
#pragma unroll
  for (int i = 0; i < kAqBlocks; ++i) {
    const int b = threadIdx.x + i * 256;
    if (b >= nb) continue;
    float bm = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) bm = fmaxf(bm, fabsf(v[i][j]));
    const uint8_t sb = (S > 0.f) ? e4m3_rne_bits(bm / (6.0f * S)) : 0;
    const float denom = e4m3_value_dev(sb) * S;
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t c = denom > 0.f ? e2m1_rne(v[i][j] / denom) : 0u;
      packed[j / 8] |= c << (4 * (j % 8));  // element 2m in the low nibble of byte m
    }
    a.scales[tok_scale_index(t, b, a.K)] = sb;
    *reinterpret_cast<uint2*>(a.codes + (size_t)t * (a.K / 2) + (size_t)b * 8) = make_uint2(packed[0], packed[1]);
  }
}

// Wide NVFP4 quantizer of a split bf16 GEMM input: one thread per 16-element block, grid
// (ceil(K / 16 / 256), T).  The row scale S = amax / (6 * 448) comes from the row's partial
// maxima (a.amax[i][t], i < n_amax), reduced by every CTA in the same order.
__global__ void __launch_bounds__(256) k_act_quant_wide(ActQuantArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[8];
  const int t = blockIdx.y, nb = a.K / 16;
  float m = 0.f;
  for (int i = threadIdx.x; i < a.n_amax; i += 256) m = fmaxf(m, a.amax[(size_t)i * a.T + t]);
  m = warp_max(m);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = m;
  __syncthreads();
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float S = amax / (6.0f * 448.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) a.sx[t] = S;
  const int b = blockIdx.x * 256 + threadIdx.x;
  if (b >= nb) return;
  const size_t off = (size_t)t * a.K + (size_t)b * 16;
  float v[16];
  float bm = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    v[j] = bf2f(a.xb[off + j]) + bf2f(a.xb[off + j + a.xb_lo]);
    bm = fmaxf(bm, fabsf(v[j]));
  }
  const uint8_t sb = (S > 0.f) ? e4m3_rne_bits(bm / (6.0f * S)) : 0;
  const float denom = e4m3_value_dev(sb) * S;
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t c = denom > 0.f ? e2m1_rne(v[j] / denom) : 0u;
    packed[j / 8] |= c << (4 * (j % 8));
  }
  a.scales[tok_scale_index(t, b, a.K)] = sb;
  *reinterpret_cast<uint2*>(a.codes + (size_t)t * (a.K / 2) + (size_t)b * 8) = make_uint2(packed[0], packed[1]);
}

// NVFP4 matrix -> bf16 values q sigma (without the tensor scale; exact in bf16), one thread
// per 16-element block.
__global__ void k_nvfp4_dequant_bf16(const uint8_t* codes, const uint8_t* scales, long n_blocks,
                                     __nv_bfloat16* out) {
  const long b = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= n_blocks) return;
  const float sig = e4m3_value_dev(scales[b]);
  __align__(16) __nv_bfloat16 o[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint8_t c = codes[b * 8 + j];
    o[2 * j] = f2bf(e2m1_value_dev(c & 15) * sig);
    o[2 * j + 1] = f2bf(e2m1_value_dev(c >> 4) * sig);
  }
  uint4* dst = reinterpret_cast<uint4*>(out + b * 16);
  dst[0] = reinterpret_cast<const uint4*>(o)[0];
  dst[1] = reinterpret_cast<const uint4*>(o)[1];
}

// Every kernel of a round prefers the largest shared-memory carve-out, the one the GEMMs run
// with: an SM can then host a GEMM CTA beside the CTAs of the kernel before it without
// reconfiguring its L1 / shared-memory split, so the GEMM's early weight loads (issued before
// its dependency wait) overlap that kernel.
int ops_init_attributes() {
  static PerDeviceOnce once;
  return once_on_current_device(once, [] {
  const void* ks[] = {(const void*)k_finish_qkv,  (const void*)k_finish_silu,   (const void*)k_finish_store,
                      (const void*)k_resid_norm,  (const void*)k_act_quant,     (const void*)k_to_bf16,
                      (const void*)k_act_quant_wide,
                      (const void*)k_rowstats_part, (const void*)k_rowstats_final, (const void*)k_commit,
                      (const void*)k_block_init,  (const void*)k_block_finish};
  for (const void* k : ks) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return (int)e;
  }
  return 0;
  });
}

}  // namespace dlm

// dlm_ops.h -- argument structs and declarations of the light kernels (dlm_ops.cu).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dlm_internal.h"

namespace dlm {

struct FinishArgs {
  GemmOut out;   // partial sums of the GEMM
  EpiArgs epi;   // op applied to each finished tile
  int N;         // valid output features
};

constexpr int kRnCluster = 4;  // CTAs per token of k_resid_norm (a thread-block cluster)

struct ResNormArgs {
  GemmOut out;                 // partial sums of a GEMM with N = d (partial == nullptr: y = 0)
  float* h;                    // [T][d] residual stream
  const __nv_bfloat16* embed;  // non-null: h = E[tokens] + y instead of h += y
  const uint8_t* embed_codes;  // or, for an NVFP4 E: its codes [V][d/2] and scales [V][d/16]
  const uint8_t* embed_sc;     //   (the rows dequantized here, q sigma, times embed_scale)
  const int32_t* tokens;       // token of row t < tok_split (all rows when tokens2 is null)
  const int32_t* tokens2;      // token of row t >= tok_split: tokens2[t - tok_split]
  int tok_split;
  float embed_scale;           // E rows are multiplied by it (1 for bf16 weights)
  const __nv_bfloat16* gain;   // [d]
  __nv_bfloat16* xn;           // [T][d] high halves
  long xn_lo;                  // elements to the low halves
  uint8_t* qcodes;             // non-null: also quantize xn to NVFP4 (see ActQuantArgs)
  uint8_t* qscales;
  float* qsx;
  int d;
  float eps;
};

struct RowStatsArgs {
  const float* logits;  // [B][ld]
  int ld;
  int V;
  int mask_id;
  int chunk;            // vocabulary entries per CTA
  float* part;          // [B][n_chunks] float4 (m, argmax bits, Z, A)
  dlm_row_stats stats;
  __nv_bfloat16* P;     // [B][V] high halves, or nullptr
  long P_lo;            // elements to the low halves, 0 = none
};

// Per-row NVFP4 quantizer of GEMM input activations: row t of x (fp32 `xf`, or the split
// bf16 pair `xb` + `xb_lo`) gets the scale sx[t] = amax / (6 * 448), one e4m3 scale sigma
// per 16 elements and e2m1 codes (codes[t][K/2], element 2j in the low nibble).  The
// scales are written in the FP4 MMA's copy layout: byte (b / 4) * 512 + t * 16 + b % 4 holds
// the scale of group b (tokens t < 32; the other 12 bytes of each 16 are not used).
struct MoeRouteArgs {
  const float* h;            // [T][d] residual rows
  const __nv_bfloat16* g;    // [d] RMSNorm gain
  const __nv_bfloat16* wr;   // [E][d] router
  float eps;
  int T, d, E, k;            // E <= 256, k <= 8, d % 8 == 0
  float* x;                  // [T][d] normalised rows
  float* logits;             // [T][E]
  float* route_w;            // [T][E] weights, zero for the experts not chosen
  int* topk_idx;             // [T][k] (optional)
  float* topk_w;             // [T][k] (optional)
};

struct ActQuantArgs {
  const float* xf;
  const __nv_bfloat16* xb;
  long xb_lo;
  int K;
  uint8_t* codes;
  uint8_t* scales;
  float* sx;
  // Wide form (k_act_quant_wide, split bf16 input): the row amax is the max of n_amax partial
  // maxima amax[i][t] (one per 64-feature tile, written by the SiLU finisher); T rows.
  const float* amax;
  int n_amax;
  int T;
};

int ops_init_attributes();

constexpr int kCommitThreads = 256;  // k_commit's block (B <= 64)

struct CommitArgs {
  const float* maxprob;
  const int32_t* argmax;
  int32_t* tokens;
  uint8_t* committed;
  float* s;
  int32_t* round;
  int32_t* status;
  int B, d;
  float tau;
  int mode, k;
  int use_cond;
  cudaGraphConditionalHandle cond;
};

struct BlockInitArgs {
  int32_t* tokens;
  uint8_t* committed;
  float* s;
  int32_t* round;
  int32_t* status;
  int B, d, mask_id;
};

struct BlockFinishArgs {
  const int32_t* tokens;
  const int32_t* round;
  const int32_t* status;
  const int* err;
  int32_t* tokens_out;
  int32_t* rounds_out;
  int* L_dev;
  int32_t* pend_tokens;  // non-null: the block's tokens are kept for its deferred KV-fill
  int B;
};

__global__ void k_finish_qkv(FinishArgs a);
__global__ void k_finish_silu(FinishArgs a);
__global__ void k_finish_store(FinishArgs a);
__global__ void k_moe_logits(MoeRouteArgs a);
__global__ void k_moe_topk(MoeRouteArgs a);
__global__ void k_resid_norm(ResNormArgs a);
__global__ void k_to_bf16(const float* x, __nv_bfloat16* y, long n, long lo, long zero_n);
__global__ void k_rowstats_part(RowStatsArgs a);
__global__ void k_rowstats_final(RowStatsArgs a);
__global__ void k_commit(CommitArgs a);
__global__ void k_block_init(BlockInitArgs a);
__global__ void k_block_finish(BlockFinishArgs a);
__global__ void k_set_int(int* p, int v);
__global__ void k_act_quant(ActQuantArgs a);
__global__ void k_act_quant_wide(ActQuantArgs a);
__global__ void k_nvfp4_dequant_bf16(const uint8_t* codes, const uint8_t* scales, long n_blocks,
                                     __nv_bfloat16* out);
__global__ void k_rope_table(float2* tab, int max_ctx, int hd, double base);
__global__ void k_amax_to_scale(float* p);
__global__ void k_amax_bf16(const __nv_bfloat16* w, long n, unsigned* amax_bits);
__global__ void k_nvfp4_quantize(const __nv_bfloat16* w, int rows, int cols, uint8_t* codes,
                                 uint8_t* scales, const unsigned* amax_bits, float* tscale);

}  // namespace dlm

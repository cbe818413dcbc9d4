// dlm_internal.h -- declarations shared by the translation units of libdlm (host side).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dlm.h"
#include "dlm_per_device.h"

namespace dlm {

// Programmatic dependent launch for every kernel of a round (default on; a debugging
// switch turns it off).  See pdl_trigger / pdl_wait in dlm_device.cuh.
extern bool g_pdl;

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// launch_k for a grid of thread-block clusters of `cluster_x` CTAs.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Runs init() once on the calling thread's current device (see PerDeviceOnce) and returns a
// cudaError_t value: kernel attributes and symbol addresses are per device.
template <class F>
inline int once_on_current_device(PerDeviceOnce& once, F init) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  const int r = once.run(dev, init);
  return r == PerDeviceOnce::kBadDevice ? (int)cudaErrorInvalidDevice : r;
}

constexpr int kSMs = 148;        // B200 streaming multiprocessors
constexpr int kTileM = 128;      // output features per GEMM tile (tcgen05 M)
constexpr int kTileK = 64;       // reduction elements per k-block (one 128-byte swizzle atom)
constexpr int kMaxTokens = 256;  // tokens per GEMM with plain bf16 activations (tcgen05 N <= 256)
constexpr int kMaxSplitTokens = 128;  // tokens per GEMM with split (hi + lo) activations
constexpr int kMaxF4Tokens = 64;      // rows per NVFP4 GEMM: two groups of 32 (MMA N = 32 each)
// Bytes of the tiled token scales of an NVFP4 GEMM input with K elements per row, kMaxF4Tokens
// rows (one plane per group of 32; see tok_scale_index).
inline size_t f4_scale_bytes(long K) { return (size_t)(kMaxF4Tokens / 32) * (size_t)(K / 64) * 512; }

// Partial-sum layout written by the GEMM: [tile][slot][TP][128] fp32, TP = T rounded up to
// 32 (token-major: the 128 rows of one token are contiguous).  Tile tau covers
// output features [128 tau, 128 tau + 128) (for the gate/up pair: gate features
// [64 tau, 64 tau + 64) in rows 0..63 and up features in rows 64..127).  The slots of a
// tile are the CTAs whose stream-K range intersects it, summed in slot order.
struct GemmOut {
  float* partial;
  int T;          // tokens
  int n_tiles;
  int n_kb;
  int grid;       // CTAs of the stream-K partition
  long units;     // n_tiles * n_kb
  int max_slots;
};

enum AMode : int {
  A_KMAJOR = 0,   // W [N][K]: one 128-row box per k-block
  A_PAIR = 1,     // two matrices [F][K] interleaved 64 + 64 rows per tile (gate/up)
  A_MNMAJOR = 2,  // A^T stored [K][N] (e.g. E [V][d] for s = P E): two 64-column boxes
};

// What the GEMM does with a finished output tile.  The CTA that completes a tile (the only
// CTA of a single-slot tile, else the last of its slots to arrive, found with a per-tile
// counter) sums the slots in slot order and applies the op; the counter is reset to zero
// for the next GEMM.
enum EpiOp : int {
  EPI_PARTIAL = 0,  // leave the per-slot partial sums only (kernel timing)
  EPI_STORE = 1,    // out[t][n] = y (fp32)
  EPI_QKV = 2,      // RoPE on q/k heads, bf16 q and K/V cache rows at position L + t
  EPI_RESID = 3,    // h[t][n] += y; ss[tile][t] = sum of h^2 over the tile's rows
  EPI_SILU = 4,     // gate/up pair: act[t][f] = silu(g) * u as a split bf16 pair
  EPI_EMBED = 5,    // h[t][n] = E[token_t][n] + y; ss[tile][t] as EPI_RESID
};

struct EpiArgs {
  int op;
  int* tile_cnt;                // [n_tiles] arrival counters, zero between GEMMs
  float* out;                   // EPI_STORE
  int ld;
  __nv_bfloat16 *q, *kc, *vc;   // EPI_QKV (bf16 K/V cache)
  uint8_t *kc8, *vc8;           // EPI_QKV with an FP8 KV cache: e4m3 rows ...
  float *ks, *vs;               // ... and their scales [Hkv][max_ctx]
  int Hq, Hkv, hd, max_ctx;
  int pos0;
  const int* pos0_dev;
  int pos_off;                  // added to *pos0_dev (graph mode): position of token 0
  const float2* rope_tab;       // (cos, sin) of position p, pair j at [p][j], j < hd/2
  float scale;                  // EPI_STORE: out = scale * y (0 means 1)
  float* h;                     // EPI_RESID / EPI_EMBED: [T][d]
  float* ss;                    // [n_tiles][T]
  const __nv_bfloat16* embed;   // EPI_EMBED
  const int32_t* tokens;
  __nv_bfloat16* act;           // EPI_SILU: [T][F] high halves
  long act_lo;
  float* act_amax;              // EPI_SILU (optional): [F / 64][T] amax of each tile's stored values
  const float* route_w;         // EPI_SILU (optional): act[t][f] *= route_w[t][f / route_f] (routed experts)
  int route_e, route_f;         //   experts per row of route_w, features per expert
  const float* add;             // EPI_STORE (optional): out = add + y (same layout as out)
};

struct GemmPlan {
  CUtensorMap ta0, ta1, tb;
  EpiArgs epi;
  int a_mode;
  int nt;            // MMA N (tokens padded to 32/64/128/256; twice the pad when split)
  int lo_col;        // split activations: MMA column of the low halves (= pad), else 0
  int N, K, T;
  const void *a0, *a1, *x;
  GemmOut out;
  size_t partial_bytes;
};

// host helpers (dlm_gemm.cu)
bool encode_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, char* err, size_t errlen);
// The same with a 128-, 64- or 0-byte swizzle (bf16 elements, L2 promotion 256 B).
bool encode_tmap_2d_swizzle(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                            uint32_t box_inner, uint32_t box_outer, int swizzle_bytes, char* err, size_t errlen);
size_t gemm_partial_bytes(int T, int N, int K, int a_mode);
// Plans y = x W^T.  `a0` is W (or Wg for A_PAIR, E for A_MNMAJOR), `a1` Wu for A_PAIR.
// split: x holds high halves in rows [0, T) and low halves in rows [pad, pad + T),
// pad = split_pad(T); the GEMM computes (hi + lo) W^T with the weight tile read once.
int split_pad(int T);
bool gemm_plan(GemmPlan* p, int a_mode, const void* a0, const void* a1, const void* x, int T,
               int N, int K, float* partial, char* err, size_t errlen, bool split = false);
cudaError_t gemm_launch(const GemmPlan& p, int* d_err, cudaStream_t s);
int gemm_init_attributes();

// NVFP4 GEMM (dlm_gemm_fp4.cu): y = Q(x) W^T with W in NVFP4 on the block-scaled FP4
// tensor cores.  x is given quantized (k_act_quant): e2m1 codes [x_rows][K/2], e4m3 scales
// tiled [K/64][32][16 B], row scales sx; the weight scales come re-tiled by nvf4_sf_tile.  Leaves
// scaled per-slot partial sums like the bf16 GEMM.  K % 256 == 0, T <= 32, x_rows >= 32.
struct GemmF4Plan {
  CUtensorMap tc0, tc1, tbc;
  int a_mode;        // A_KMAJOR, or A_PAIR (gate/up: w0 = gate, w1 = up)
  int N, K, T;
  float sw0, sw1;
  const float* sx;
  const uint8_t* sfa, *sfb;
  GemmOut out;
  size_t partial_bytes;
};
size_t gemm_fp4_partial_bytes(int T, int N, int K, int a_mode);
size_t nvf4_sf_tile_bytes(int N, int K, int a_mode);
cudaError_t nvf4_sf_tile(const dlm_nvfp4_matrix& w0, const dlm_nvfp4_matrix* w1, int N, int K, int a_mode,
                         uint8_t* out, cudaStream_t s);
bool gemm_fp4_plan(GemmF4Plan* p, int a_mode, const dlm_nvfp4_matrix& w0, const dlm_nvfp4_matrix* w1,
                   const uint8_t* sfa_tiled, const uint8_t* xcodes, const uint8_t* xscales, int x_rows, const float* sx,
                   int T, int N, int K, float* partial, char* err, size_t errlen);
cudaError_t gemm_fp4_launch(const GemmF4Plan& p, int* d_err, cudaStream_t s);
int gemm_fp4_init_attributes();

// LM head fused with the row statistics and s = P E (dlm_lmhead.cu), one pass over E.
// x2: split bf16 pair of x2_rows rows of d: the T high halves start at row hi_row, the T low
// halves at row lo_row (both multiples of 8; the 32 rows from each are read, those past T
// dropped, those past x2_rows read as zeros);
// p_given: bf16 [T][V] or nullptr (P = softmax of the logits).  T <= 32, d % 256 == 0,
// d <= 3072.
bool lmhead_fused_supported(int T, int d);
size_t lmhead_fused_scratch_bytes(int V, int d);
cudaError_t lmhead_fused_launch(const void* x2, int x2_rows, int hi_row, int lo_row, const void* E,
                                const void* p_given, int T, int V, int d, int mask_id, dlm_row_stats stats,
                                float* s, void* scratch, int* d_err, cudaStream_t st, char* err,
                                size_t errlen);

// The same pass with NVFP4 E (codes [V][d/2], e4m3 scales [V][d/16], tensor scale; sfe_tiled
// its scales re-tiled by nvf4_sf_tile) and x quantized by the last RMSNorm (codes [x_rows][d/2],
// tiled scales, row scales sx): the T rows from row x_row0 (a multiple of 32: the rows of a
// round that carries a pending block start at 32).  T <= 32, d % 512 == 0, d <= 2560.
bool lmhead_fused_f4_supported(int T, int d);
cudaError_t lmhead_fused_f4_launch(const dlm_nvfp4_matrix& E, const uint8_t* sfe_tiled, const uint8_t* xcodes,
                                   int x_rows, int x_row0, const uint8_t* xscales, const float* sx, int T, int V,
                                   int d, int mask_id, dlm_row_stats stats, float* s, void* scratch, int* d_err,
                                   cudaStream_t st, char* err, size_t errlen);
// 2-D tensor map of a byte matrix [outer][inner] (rows of `inner` bytes).
bool encode_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                  uint32_t box_outer, bool swizzle128, char* err, size_t errlen);

// attention (dlm_attention.cu)
struct AttnArgs {
  const __nv_bfloat16* q;    // [T][Hq][hd]
  const __nv_bfloat16* kc;   // [Hkv][max_ctx][hd] (one layer; e4m3 bytes when ks != nullptr)
  const __nv_bfloat16* vc;
  const float* ks;           // FP8 KV cache: K / V row scales [Hkv][max_ctx], else nullptr
  const float* vs;
  __nv_bfloat16* o;          // [T][Hq][hd] (high halves when o_lo != 0)
  long o_lo;                 // elements to the low halves of a split output, 0 = plain bf16
  float* part_o;             // [max_splits][Hkv * T * G][hd]
  float* part_ml;            // [max_splits][Hkv * T * G][2]
  int T, Hq, Hkv, hd, max_ctx;
  int pos0;                  // position of query 0 when pos0_dev == nullptr
  const int* pos0_dev;       // device prefix length (graph mode); query 0 at *pos0_dev + pos_off
  int pos_off;
  int causal;                // query t sees keys [0, pos0 + t]
  int blk;                   // causal == 0: query t sees keys [0, pos0 + min(T, (t / blk + 1) blk));
                             // blk == 0 or T: every query sees [0, pos0 + T) (one block)
  int max_splits;
  int* err;
};
size_t attention_scratch_bytes(int T, int Hq, int hd, int max_splits);
int attention_max_splits(int T, int Hq, int Hkv, int max_ctx);
cudaError_t attention_launch(const AttnArgs& a, cudaStream_t s);
int attention_init_attributes();
int attention_split_cap(int T, int max_ctx);

}  // namespace dlm

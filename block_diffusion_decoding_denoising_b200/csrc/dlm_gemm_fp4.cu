// dlm_gemm_fp4.cu -- the weight-streaming GEMM for NVFP4 weights on the FP4 tensor cores:
// y = Q(x) W^T, where W is stored as e2m1 codes with one e4m3 scale per 16 consecutive
// elements of a row and an fp32 tensor scale, and Q quantizes each row of x to the same
// format (k_act_quant).
//
// The pages ("ORL: diffusion LLMs get a learnable 'tokens per forward'", section "What
// shipped": the B200 and RTX 5090 numbers are NVFP4) give only the format; the kernel is
// this library's own design.  tcgen05.mma kind::mxf4nvf4 with 16-element block scaling
// multiplies e2m1 codes from shared memory and applies the e4m3 block scales of both
// operands, which it reads from tensor memory:
//   y[t][n] = S_w S_x[t] sum_k (q_w sigma_w)[n][k] (q_x sigma_x)[t][k]
// with the two fp32 tensor scales applied in the epilogue.
//
// Per CTA (192 threads): warp 0 TMA producer, warp 1 MMA issuer, warps 2..5 epilogue.  A
// stage holds 256 reduction elements: the codes of a 128-row weight tile (16 KB, 128-byte
// swizzle), the codes of 32 tokens (4 KB), the weight tile's scales (2 KB, pre-tiled, see
// below) and the tokens' scales (2 KB, pre-tiled).  The MMA thread copies the scales into tensor
// memory (tcgen05.cp, 32 lanes x 128 bits, replicated to the four lane quarters) and issues
// four K = 64 MMAs per stage.  Inputs of 33..64 rows (a round carrying a pending block) run as
// two groups of 32 tokens: a stage then holds both groups' codes and scales (30 KB, 7 stages)
// and each group issues its own four N = 32 MMAs on the shared weight tile, into its own half
// of the accumulator.  Work is cut stream-K over (tile, 256-element k-block) units
// exactly like the bf16 GEMM, and the epilogue writes scaled partial sums in the same
// [tile][slot][TP][128] layout, so the same finish kernels complete it.
//
// Scale layout in tensor memory (one K = 64 MMA): the scale of row m (of 128) and 16-element
// group k (of 4) sits in lane m % 32 of every lane quarter, 32-bit column m / 32, byte k; the
// 32 tokens' scales in lane t, one column.  Each MMA's scales get their own 4-column slot.
// The weight scales are therefore re-tiled once (k_sf_tile) into [tile][64-element block]
// [lane 32][column 4][byte 4], and the quantizer writes the token scales as [group of 32
// tokens][64-element block][token % 32][16 B] (4 bytes used; tok_scale_index), so that a
// stage's four blocks of one group are 2 KB of contiguous 512-byte copy sources.
#include <cuda_fp16.h>
#include <stdio.h>
#include <string.h>

#include "dlm_device.cuh"
#include "dlm_internal.h"

namespace dlm {

namespace {

constexpr int kF4K = 256;          // reduction elements per stage (128 code bytes per row)
constexpr int kF4Mmas = kF4K / 64; // K = 64 MMAs per stage
constexpr int kF4ACodes = kTileM * 128;   // 16 KB
constexpr int kF4BCodes = 32 * 128;       // 4 KB per group of 32 tokens
constexpr int kF4SfA = kTileM * kF4K / 16;  // 2 KB
constexpr int kF4SfB = kF4Mmas * 32 * 16;  // 2 KB per group: per MMA 32 tokens x 16 B (4 scale bytes used)
constexpr int kF4TmemCols = 512;
// Stage layout for G groups of 32 tokens (G = 1: up to 32 rows; G = 2: up to 64, the rows of
// a round that carries a pending block): weight codes | G token-code boxes | weight scales |
// G token-scale blocks.  Each group runs its own four N = 32 MMAs on the shared weight tile.
template <int G>
struct F4Cfg {
  static constexpr int kOffB = kF4ACodes;
  static constexpr int kOffSfA = kOffB + G * kF4BCodes;
  static constexpr int kOffSfB = kOffSfA + kF4SfA;
  static constexpr int kStageBytes = kOffSfB + G * kF4SfB;  // 24 KB / 30 KB
  static constexpr int kStages = G == 1 ? 8 : 7;
  static constexpr int kSmem = kStages * kStageBytes + 1024 + 512;
  static constexpr int kAccCols = G * 32;                  // one accumulator (all groups)
  static constexpr int kSfCol = 2 * kAccCols;              // two accumulators, then the scales
  // per stage and MMA, a 4-column slot for the weight scales and one per group for the tokens'
  static constexpr int kSfColsPerStage = 4 * kF4Mmas * (1 + G);
};
static_assert(F4Cfg<1>::kStageBytes == 24576 && F4Cfg<2>::kStageBytes == 30720, "stage layout");
static_assert(F4Cfg<2>::kSmem <= 232448, "nvfp4 gemm shared memory");
static_assert(F4Cfg<1>::kSfCol + F4Cfg<1>::kStages * F4Cfg<1>::kSfColsPerStage <= kF4TmemCols, "tmem budget");
static_assert(F4Cfg<2>::kSfCol + F4Cfg<2>::kStages * F4Cfg<2>::kSfColsPerStage <= kF4TmemCols, "tmem budget");

struct F4KArgs {
  int a_mode;        // A_KMAJOR or A_PAIR
  int T;
  GemmOut out;
  float sw0, sw1;    // tensor scales (rows 0..63 / 64..127 of a pair tile use sw0 / sw1)
  const float* sx;   // [T] row scales of the quantized activations
  const uint8_t* sfa;  // tiled weight scales (k_sf_tile)
  const uint8_t* sfb;  // tiled token scales (k_act_quant): group g's plane at sfb + g * K / 64 * 512
  int nb64;            // K / 64
  int* err;
};

__device__ __forceinline__ void epi_sync_f4() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int G>
__global__ void __launch_bounds__(192, 1)
k_gemm_nvf4(const __grid_constant__ CUtensorMap tc0, const __grid_constant__ CUtensorMap tc1,
            const __grid_constant__ CUtensorMap tbc, F4KArgs args) {
  using Cf = F4Cfg<G>;
  constexpr int S = Cf::kStages;
  constexpr int kF4StageBytes = Cf::kStageBytes;
  constexpr int kF4OffB = Cf::kOffB, kF4OffSfA = Cf::kOffSfA, kF4OffSfB = Cf::kOffSfB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + S * kF4StageBytes);
  uint64_t* full = bars;                    // [S]
  uint64_t* empty = bars + S;               // [S]
  uint64_t* acc_full = bars + 2 * S;        // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* mma_done = acc_empty + 2;       // [1]
  uint32_t* tmem_holder = (uint32_t*)(mma_done + 1);
  int* flag = (int*)(mma_done + 2);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const GemmOut& o = args.out;
  const int c = blockIdx.x;
  const long u_begin = unit_begin(c, o.units, o.grid), u_end = unit_begin(c + 1, o.units, o.grid);

  if (warp == 1 && lane == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 128); }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, kF4TmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tc0);
    if (args.a_mode == A_PAIR) prefetch_tmap(&tc1);
    prefetch_tmap(&tbc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  if (warp != 0) pdl_wait();

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    uint32_t armed_parity[S];
    bool armed[S];
    for (int i = 0; i < S; ++i) armed[i] = false;
    auto load_w = [&](long u, int st) {  // weight codes and tiled weight scales
      const int tile = (int)(u / o.n_kb), kb = (int)(u % o.n_kb);
      uint8_t* base = smem + st * kF4StageBytes;
      if (args.a_mode == A_PAIR) {
        tma_load_2d(base, &tc0, &full[st], kb * 128, tile * 64);
        tma_load_2d(base + kF4ACodes / 2, &tc1, &full[st], kb * 128, tile * 64);
      } else {
        tma_load_2d(base, &tc0, &full[st], kb * 128, tile * kTileM);
      }
      bulk_load(base + kF4OffSfA, args.sfa + ((size_t)tile * o.n_kb + kb) * kF4SfA, kF4SfA, &full[st]);
    };
    auto load_x = [&](long u, int st) {  // token codes and tiled token scales, per group
      const int kb = (int)(u % o.n_kb);
      uint8_t* base = smem + st * kF4StageBytes;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        tma_load_2d(base + kF4OffB + g * kF4BCodes, &tbc, &full[st], kb * 128, g * 32);
        bulk_load(base + kF4OffSfB + g * kF4SfB, args.sfb + ((size_t)g * args.nb64 + (size_t)kb * kF4Mmas) * 512,
                  kF4SfB, &full[st]);
      }
    };
    const long n_pre = (u_end - u_begin) < S ? (u_end - u_begin) : S;
    for (long i = 0; i < n_pre; ++i) {
      mbar_arrive_expect_tx(&full[i], kF4StageBytes);
      armed[i] = true;
      armed_parity[i] = 0;
      load_w(u_begin + i, (int)i);
    }
    pdl_wait();
    for (long i = 0; i < n_pre; ++i) load_x(u_begin + i, (int)i);
    int stage = (int)(n_pre % S);
    uint32_t phase = (n_pre == S) ? 1u : 0u;
    for (long u = u_begin + n_pre; u < u_end; ++u) {
      if (!mbar_wait(&empty[stage], phase ^ 1, args.err)) break;
      mbar_arrive_expect_tx(&full[stage], kF4StageBytes);
      armed[stage] = true;
      armed_parity[stage] = phase;
      load_w(u, stage);
      load_x(u, stage);
      if (++stage == S) { stage = 0; phase ^= 1; }
    }
    pdl_trigger();
    for (int i = 0; i < S; ++i)
      if (armed[i]) mbar_wait(&full[i], armed_parity[i], args.err);
  } else if (warp == 1) {
    // ---------------- MMA issuer: scales to TMEM, four K = 64 block-scaled MMAs per stage.
    // The whole warp runs the loop and waits (outcomes made warp-uniform); one elected lane
    // issues the copies, the MMAs and the commits.
    constexpr uint32_t idesc = idesc_nvf4(128, 32);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    long u = u_begin;
    while (u < u_end && ok) {
      const int tile = (int)(u / o.n_kb);
      const long seg_end = ((long)tile + 1) * o.n_kb < u_end ? ((long)tile + 1) * o.n_kb : u_end;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_empty[acc], acc_phase ^ 1, args.err))) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * Cf::kAccCols;
      for (long uu = u; uu < seg_end; ++uu) {
        if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, args.err))) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * kF4StageBytes);
        const uint32_t sfa_col = tmem_base + Cf::kSfCol + stage * Cf::kSfColsPerStage;
        const uint32_t sfb_col = sfa_col + 4 * kF4Mmas;  // + 16 columns per group
        const uint64_t ad = sw128_desc(sa, 16, 1024);
        const uint64_t fa = sf_desc(sa + kF4OffSfA);
        if (elect_one()) {
#pragma unroll
          for (int j = 0; j < kF4Mmas; ++j) {  // +512 B per copy source
            tmem_cp_32x128(sfa_col + 4 * j, fa + 32 * j);
#pragma unroll
            for (int g = 0; g < G; ++g)
              tmem_cp_32x128(sfb_col + 16 * g + 4 * j, sf_desc(sa + kF4OffSfB + g * kF4SfB) + 32 * j);
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const uint64_t bd = sw128_desc(sa + kF4OffB + g * kF4BCodes, 16, 1024);
#pragma unroll
            for (int j = 0; j < kF4Mmas; ++j)  // +32 B per K = 64 step
              mma_nvf4(d_tmem + 32 * g, ad + 2 * j, bd + 2 * j, idesc, sfa_col + 4 * j, sfb_col + 16 * g + 4 * j,
                       (uu > u || j > 0) ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&acc_full[acc]);
      __syncwarp();
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      u = seg_end;
    }
    if (elect_one()) {
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, args.err);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> scaled partial sums
    const int quarter = warp % 4;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64;
    const float sw = (args.a_mode == A_PAIR && row >= 64) ? args.sw1 : args.sw0;
    const int TP = G * 32;
    int acc = 0;
    uint32_t acc_phase = 0;
    long u = u_begin;
    float v[32];
    while (u < u_end) {
      const int tile = (int)(u / o.n_kb);
      const long seg_end = ((long)tile + 1) * o.n_kb < u_end ? ((long)tile + 1) * o.n_kb : u_end;
      if (et == 0) *flag = mbar_wait(&acc_full[acc], acc_phase, args.err) ? 1 : 0;
      epi_sync_f4();
      const bool got = *flag != 0;
      epi_sync_f4();
      if (!got) break;
      tc_fence_after();
      const int lo_c = cta_of_unit((long)tile * o.n_kb, o.units, o.grid);
      const int slot = c - lo_c;
      float* dst = o.partial + ((size_t)tile * o.max_slots + slot) * kTileM * TP + row;
#pragma unroll 1
      for (int g = 0; g < G; ++g) {
        tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * Cf::kAccCols + 32 * g, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = 32 * g + j;
          dst[(size_t)t * kTileM] = (t < args.T) ? v[j] * (sw * args.sx[t]) : 0.f;
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      u = seg_end;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, kF4TmemCols);
}

// Re-tiles weight scales [rows][K/16] into [tile][K/64][lane 32][column 4][byte 4]: byte
// (l, c, k) of block (tile, b) is the scale of tile row 32 c + l, 16-element group 4 b + k.
// Pair tiles take rows 0..63 from s0 (rows 64 tile ..) and rows 64..127 from s1.  Rows past
// N get scale 0.  One thread per 4-byte group (l, c) of a block.
__global__ void k_sf_tile(const uint8_t* s0, const uint8_t* s1, int N, int K, int pair, int n_tiles,
                          uint8_t* out) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;  // (tile, b, l, c)
  const int nb = K / 64;
  const long total = (long)n_tiles * nb * 128;
  if (i >= total) return;
  const int cl = (int)(i % 128), b = (int)((i / 128) % nb), tile = (int)(i / (128L * nb));
  const int l = cl / 4, col = cl % 4;
  const int r = 32 * col + l;  // tile row
  const uint8_t* src;
  int grow;
  if (pair) {
    src = r < 64 ? s0 : s1;
    grow = tile * 64 + (r & 63);
  } else {
    src = s0;
    grow = tile * kTileM + r;
  }
  uint32_t w = 0;
  if (grow < N) {
    const uint8_t* p = src + (size_t)grow * (K / 16) + 4 * b;
    w = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
  }
  reinterpret_cast<uint32_t*>(out)[i] = w;
}

typedef CUresult (*PFN_encodeTiledF4)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                      CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw, char* err,
               size_t errlen) {
  static PFN_encodeTiledF4 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_encodeTiledF4)p;
  }
  if (!fn) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled entry point unavailable");
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled failed (%d): dims %llu x %llu box %u x %u", (int)r,
             (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
    return false;
  }
  return true;
}

void partition_f4(int T, int N, int K, int a_mode, GemmOut* o) {
  const int rows_per_tile = (a_mode == A_PAIR) ? 64 : kTileM;
  o->T = T;
  o->n_tiles = (N + rows_per_tile - 1) / rows_per_tile;
  o->n_kb = K / kF4K;
  o->units = (long)o->n_tiles * o->n_kb;
  o->grid = o->units < kSMs ? (int)o->units : kSMs;
  int ms = 1;
  for (int t = 0; t < o->n_tiles; ++t) {
    int lo = cta_of_unit((long)t * o->n_kb, o->units, o->grid);
    int hi = cta_of_unit((long)(t + 1) * o->n_kb - 1, o->units, o->grid);
    if (hi - lo + 1 > ms) ms = hi - lo + 1;
  }
  o->max_slots = ms;
}

}  // namespace

bool encode_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                  uint32_t box_outer, bool swizzle128, char* err, size_t errlen) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, outer, inner, box_inner, box_outer,
                   swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, err, errlen);
}

size_t gemm_fp4_partial_bytes(int T, int N, int K, int a_mode) {
  GemmOut o;
  partition_f4(T, N, K, a_mode, &o);
  return (size_t)o.n_tiles * o.max_slots * ((T + 31) / 32 * 32) * kTileM * sizeof(float);
}

size_t nvf4_sf_tile_bytes(int N, int K, int a_mode) {
  const int rows = (a_mode == A_PAIR) ? 64 : kTileM;
  return (size_t)((N + rows - 1) / rows) * (K / 64) * 512;
}

cudaError_t nvf4_sf_tile(const dlm_nvfp4_matrix& w0, const dlm_nvfp4_matrix* w1, int N, int K, int a_mode,
                         uint8_t* out, cudaStream_t s) {
  const int rows = (a_mode == A_PAIR) ? 64 : kTileM;
  const int n_tiles = (N + rows - 1) / rows;
  const long total = (long)n_tiles * (K / 64) * 128;
  k_sf_tile<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
      (const uint8_t*)w0.scales, w1 ? (const uint8_t*)w1->scales : nullptr, N, K, a_mode == A_PAIR ? 1 : 0, n_tiles,
      out);
  return cudaGetLastError();
}

bool gemm_fp4_plan(GemmF4Plan* p, int a_mode, const dlm_nvfp4_matrix& w0, const dlm_nvfp4_matrix* w1,
                   const uint8_t* sfa_tiled, const uint8_t* xcodes, const uint8_t* xscales, int x_rows, const float* sx,
                   int T, int N, int K, float* partial, char* err, size_t errlen) {
  memset(p, 0, sizeof(*p));
  if (T < 1 || T > kMaxF4Tokens || N < 1 || K < kF4K || K % kF4K != 0 || x_rows < 32 ||
      (a_mode != A_KMAJOR && a_mode != A_PAIR) || (a_mode == A_PAIR && !w1) || !w0.codes || !sfa_tiled ||
      (w1 && !w1->codes) || !xcodes || !xscales || !sx) {
    snprintf(err, errlen, "nvfp4 gemm: unsupported arguments T=%d N=%d K=%d (K must be a multiple of %d, T <= %d)",
             T, N, K, kF4K, kMaxF4Tokens);
    return false;
  }
  p->a_mode = a_mode;
  p->T = T;
  p->N = N;
  p->K = K;
  p->sw0 = w0.tensor_scale;
  p->sw1 = w1 ? w1->tensor_scale : w0.tensor_scale;
  p->sx = sx;
  p->sfa = sfa_tiled;
  partition_f4(T, N, K, a_mode, &p->out);
  p->out.partial = partial;
  if ((unsigned long long)p->out.units * (unsigned long long)p->out.grid >= (1ull << 32)) {
    snprintf(err, errlen, "gemm: %ld units exceed the 32-bit partition arithmetic", p->out.units);
    return false;
  }
  p->partial_bytes = gemm_fp4_partial_bytes(T, N, K, a_mode);
  const uint32_t rows = (a_mode == A_PAIR) ? 64 : kTileM;
  bool ok = encode_2d(&p->tc0, CU_TENSOR_MAP_DATA_TYPE_UINT8, w0.codes, (uint64_t)K / 2, N, (uint64_t)K / 2, 128,
                      rows, CU_TENSOR_MAP_SWIZZLE_128B, err, errlen);
  if (ok && a_mode == A_PAIR)
    ok = encode_2d(&p->tc1, CU_TENSOR_MAP_DATA_TYPE_UINT8, w1->codes, (uint64_t)K / 2, N, (uint64_t)K / 2, 128, rows,
                   CU_TENSOR_MAP_SWIZZLE_128B, err, errlen);
  else
    p->tc1 = p->tc0;
  // token codes [x_rows][K/2] (128-byte swizzle); token scales tiled (k_act_quant)
  p->sfb = xscales;
  // (all x_rows rows: a 64-row input is loaded as two 32-row boxes)
  ok = ok && encode_2d(&p->tbc, CU_TENSOR_MAP_DATA_TYPE_UINT8, xcodes, (uint64_t)K / 2, (uint64_t)x_rows,
                       (uint64_t)K / 2, 128, 32, CU_TENSOR_MAP_SWIZZLE_128B, err, errlen);
  return ok;
}

cudaError_t gemm_fp4_launch(const GemmF4Plan& p, int* d_err, cudaStream_t s) {
  F4KArgs a;
  a.a_mode = p.a_mode;
  a.T = p.T;
  a.out = p.out;
  a.sw0 = p.sw0;
  a.sw1 = p.sw1;
  a.sx = p.sx;
  a.sfa = p.sfa;
  a.sfb = p.sfb;
  a.nb64 = p.K / 64;
  a.err = d_err;
  if (p.T > 32)
    return launch_k(k_gemm_nvf4<2>, dim3(p.out.grid), dim3(192), F4Cfg<2>::kSmem, s, p.tc0, p.tc1, p.tbc, a);
  return launch_k(k_gemm_nvf4<1>, dim3(p.out.grid), dim3(192), F4Cfg<1>::kSmem, s, p.tc0, p.tc1, p.tbc, a);
}

int gemm_fp4_init_attributes() {
  static PerDeviceOnce once;
  return once_on_current_device(once, [] {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_nvf4<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, F4Cfg<1>::kSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_gemm_nvf4<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, F4Cfg<2>::kSmem);
    return (int)e;
  });
}

}  // namespace dlm

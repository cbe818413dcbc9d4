// dlm_gemm_fp4.cu -- the weight-streaming GEMM for NVFP4 weights: y = x W^T where W is
// stored as e2m1 codes with one e4m3 scale per 16 consecutive elements of a row and an
// fp32 tensor scale, and x is quantized per row to the same format.
//
// The pages ("ORL: diffusion LLMs get a learnable 'tokens per forward'", section "What
// shipped": the B200 and RTX 5090 numbers are NVFP4) give only the format; the kernel is
// this library's own design.  A weight code times its block scale (q sigma) has at most
// 6 significant bits and lies in [2^-10, 2688], so it is exact in f16; the same holds for
// the quantized activations.  The tensor cores therefore see exact f16 operands, and
//   y[t][n] = S_w S_x[t] sum_k (q_w sigma_w)[n][k] (q_x sigma_x)[t][k]
// equals the product of the dequantised operands up to fp32 accumulation order.
//
// Per CTA (320 threads): warp 0 TMA producer, warp 1 MMA issuer, warps 2..5 epilogue,
// warps 6..9 decoders.  A stage holds 256 reduction elements of a 128-row weight tile
// (16 KB of codes, 2 KB of scales) and of the activations (4 x 64-element boxes).  Each
// decoder thread owns one weight row (= one TMEM lane): it turns its 128 code bytes into
// f16 pairs, multiplies by the block scale and stores 64-element sub-blocks straight into
// tensor memory (tcgen05.st), where the MMA reads the A operand.  The decoded tile never
// goes through shared memory.  Work is cut stream-K over (tile, 256-element k-block) units
// exactly like the bf16 GEMM, and the epilogue writes scaled partial sums in the same
// [tile][slot][TP][128] layout, so the same finish kernels complete it.
#include <cuda_fp16.h>
#include <stdio.h>
#include <string.h>

#include "dlm_device.cuh"
#include "dlm_internal.h"

namespace dlm {

namespace {

constexpr int kF4K = 256;            // reduction elements per stage (128 code bytes per row)
constexpr int kSubs = kF4K / 64;     // 64-element sub-blocks per stage
constexpr int kASlots = 8;           // decoded A sub-blocks resident in tensor memory (two stages)
constexpr int kACol = 128;           // first TMEM column of the A slots (32 columns each)
static_assert(kASlots % kSubs == 0, "a stage's sub-blocks take consecutive slots");
constexpr int kF4Threads = 320;

template <int NT>
struct F4Cfg {
  static constexpr int kCodeBytes = kTileM * 128;   // 16 KB, 128-byte swizzled rows
  static constexpr int kBSub = NT * 128;            // one 64-element box of NT f16 rows
  static constexpr int kBBytes = kSubs * kBSub;
  static constexpr int kScaleBytes = kTileM * 16;   // 2 KB
  static constexpr int kStageBytes = kCodeBytes + kBBytes + kScaleBytes;  // multiple of 1024
  static constexpr int kStages = NT <= 32 ? 6 : 4;
  static constexpr int kSmem = kStages * kStageBytes + 1024 /*align*/ + 512 /*barriers*/;
  static constexpr int kTmemCols = 512;             // 2 accumulators (<= 128) + A slots
};

struct F4KArgs {
  int a_mode;        // A_KMAJOR or A_PAIR
  int T;
  GemmOut out;
  float sw0, sw1;    // tensor scales (rows 0..63 / 64..127 of a pair tile use sw0 / sw1)
  const float* sx;   // [T] row scales of the quantized activations
  int* err;
};

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16 with f16 inputs.
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f16 with f16 A/B (format 0), fp32 D, K-major operands.
__host__ __device__ constexpr uint32_t idesc_f16(int m, int n) {
  return (1u << 4) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

// Four bytes of e2m1 code pairs -> four f16x2 words (the low nibble of a byte is the
// element of lower index and lands in the low half).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t codes, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, c0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, c1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, c2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, c3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(codes));
}

// Four e4m3 scale bytes -> each scale as a broadcast f16x2 pair.
__device__ __forceinline__ void e4m3x4_to_f16x2_bcast(uint32_t sc, uint32_t (&s)[4]) {
  uint32_t lo, hi;
  asm("{\n\t.reg .b16 a, b;\n\t"
      "mov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(sc));
  s[0] = __byte_perm(lo, 0, 0x1010);
  s[1] = __byte_perm(lo, 0, 0x3232);
  s[2] = __byte_perm(hi, 0, 0x1010);
  s[3] = __byte_perm(hi, 0, 0x3232);
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ void epi_sync_f4() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int NT>
__global__ void __launch_bounds__(kF4Threads, 1)
k_gemm_fp4(const __grid_constant__ CUtensorMap tc0, const __grid_constant__ CUtensorMap tc1,
           const __grid_constant__ CUtensorMap ts0, const __grid_constant__ CUtensorMap ts1,
           const __grid_constant__ CUtensorMap tb, F4KArgs args) {
  using Cfg = F4Cfg<NT>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + S * Cfg::kStageBytes);
  uint64_t* full = bars;                    // [S]  TMA bytes of a stage landed
  uint64_t* empty = bars + S;               // [S]  MMAs of a stage done
  uint64_t* a_full = bars + 2 * S;          // [4]  decoded sub-block stored in TMEM
  uint64_t* a_empty = a_full + kASlots;     // [4]  MMAs reading a slot done
  uint64_t* acc_full = a_empty + kASlots;   // [2]
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
    for (int i = 0; i < kASlots; ++i) { mbar_init(&a_full[i], 4); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 128); }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tc0);
    prefetch_tmap(&ts0);
    if (args.a_mode == A_PAIR) { prefetch_tmap(&tc1); prefetch_tmap(&ts1); }
    prefetch_tmap(&tb);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  if (warp != 0) pdl_wait();

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    uint32_t armed_parity[8];
    bool armed[8];
    for (int i = 0; i < S; ++i) armed[i] = false;
    auto load_w = [&](long u, int st) {
      const int tile = (int)(u / o.n_kb), kb = (int)(u % o.n_kb);
      uint8_t* base = smem + st * Cfg::kStageBytes;
      uint8_t* sc = base + Cfg::kCodeBytes + Cfg::kBBytes;
      if (args.a_mode == A_PAIR) {
        tma_load_2d(base, &tc0, &full[st], kb * 128, tile * 64);
        tma_load_2d(base + Cfg::kCodeBytes / 2, &tc1, &full[st], kb * 128, tile * 64);
        tma_load_2d(sc, &ts0, &full[st], kb * 16, tile * 64);
        tma_load_2d(sc + Cfg::kScaleBytes / 2, &ts1, &full[st], kb * 16, tile * 64);
      } else {
        tma_load_2d(base, &tc0, &full[st], kb * 128, tile * kTileM);
        tma_load_2d(sc, &ts0, &full[st], kb * 16, tile * kTileM);
      }
    };
    auto load_x = [&](long u, int st) {
      const int kb = (int)(u % o.n_kb);
      uint8_t* sb = smem + st * Cfg::kStageBytes + Cfg::kCodeBytes;
#pragma unroll
      for (int j = 0; j < kSubs; ++j) tma_load_2d(sb + j * Cfg::kBSub, &tb, &full[st], kb * kF4K + j * 64, 0);
    };
    const long n_pre = (u_end - u_begin) < S ? (u_end - u_begin) : S;
    for (long i = 0; i < n_pre; ++i) {
      mbar_arrive_expect_tx(&full[i], Cfg::kStageBytes);
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
      mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
      armed[stage] = true;
      armed_parity[stage] = phase;
      load_w(u, stage);
      load_x(u, stage);
      if (++stage == S) { stage = 0; phase ^= 1; }
    }
    pdl_trigger();
    for (int i = 0; i < S; ++i)
      if (armed[i]) mbar_wait(&full[i], armed_parity[i], args.err);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc = idesc_f16(128, NT);
    int stage = 0, slot = 0, acc = 0;
    uint32_t phase = 0, sphase = 0, acc_phase = 0;
    bool ok = true;
    long u = u_begin;
    while (u < u_end && ok) {
      const int tile = (int)(u / o.n_kb);
      const long seg_end = ((long)tile + 1) * o.n_kb < u_end ? ((long)tile + 1) * o.n_kb : u_end;
      if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, args.err)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * NT;
      for (long uu = u; uu < seg_end && ok; ++uu) {
        if (!mbar_wait(&full[stage], phase, args.err)) { ok = false; break; }
        const uint32_t sb = smem_u32(smem + stage * Cfg::kStageBytes + Cfg::kCodeBytes);
        for (int j = 0; j < kSubs; ++j) {
          if (!mbar_wait(&a_full[slot], sphase, args.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + kACol + slot * 32;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t bdesc = sw128_desc(sb + j * Cfg::kBSub + k * 32, 16, 1024);
            mma_f16_tmem_a(d_tmem, a_tmem + k * 8, bdesc, idesc, (uu > u || j > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&a_empty[slot]);
          if (++slot == kASlots) { slot = 0; sphase ^= 1; }
        }
        if (!ok) break;
        mma_commit(&empty[stage]);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      mma_commit(&acc_full[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      u = seg_end;
    }
    mma_commit(mma_done);
    mbar_wait(mma_done, 0, args.err);
  } else if (warp >= 6) {
    // ---------------- decoders: codes and scales of one weight row -> f16 (q sigma) in TMEM
    const int quarter = warp % 4;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16) + kACol;
    int stage = 0, slot = 0;
    uint32_t phase = 0, sphase = 0;
    bool ok = true;
    for (long u = u_begin; u < u_end && ok; ++u) {
      if (!mbar_wait(&full[stage], phase, args.err)) break;
      const uint8_t* base = smem + stage * Cfg::kStageBytes;
      uint4 cw[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)  // 16-byte chunk q of the row sits at chunk q ^ (row % 8)
        cw[q] = *reinterpret_cast<const uint4*>(base + row * 128 + ((q ^ (row & 7)) << 4));
      const uint4 scw = *reinterpret_cast<const uint4*>(base + Cfg::kCodeBytes + Cfg::kBBytes + row * 16);
      // the stage's four slots (kASlots is a multiple of kSubs: they are consecutive)
      const int slot0 = slot;
      for (int j = 0; j < kSubs && ok; ++j)
        if (!mbar_wait(&a_empty[slot0 + j], sphase ^ 1, args.err)) ok = false;
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < kSubs; ++j) {
        // sub-block j: elements 64 j .. 64 j + 63 = code chunks 2j, 2j+1, scale bytes 4j .. 4j+3
        const uint32_t sw = (j == 0) ? scw.x : (j == 1) ? scw.y : (j == 2) ? scw.z : scw.w;
        uint32_t sig[4];
        e4m3x4_to_f16x2_bcast(sw, sig);
        const uint4 c0 = cw[2 * j], c1 = cw[2 * j + 1];
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint32_t r[32];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          uint32_t h[4];
          e2m1x8_to_f16x2(words[w], h);
#pragma unroll
          for (int i = 0; i < 4; ++i) r[4 * w + i] = hmul2_u32(h[i], sig[w / 2]);  // 16 elements per scale
        }
        tmem_st32(lane_base + (slot0 + j) * 32, r);
      }
      tmem_wait_st();  // one wait for the stage's four stores
      tc_fence_before();
      __syncwarp();
      if (lane == 0)
        for (int j = 0; j < kSubs; ++j) mbar_arrive(&a_full[slot0 + j]);
      slot += kSubs;
      if (slot == kASlots) { slot = 0; sphase ^= 1; }
      if (++stage == S) { stage = 0; phase ^= 1; }
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> scaled partial sums
    const int quarter = warp % 4;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64;
    const float sw = (args.a_mode == A_PAIR && row >= 64) ? args.sw1 : args.sw0;
    const int ncb = (args.T + 31) / 32;
    const int TP = ncb * 32;
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
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * NT;
      float* dst = o.partial + ((size_t)tile * o.max_slots + slot) * kTileM * TP + row;
#pragma unroll 1
      for (int cb = 0; cb < ncb; ++cb) {
        tmem_ld32(taddr + cb * 32, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = cb * 32 + j;
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
  if (warp == 0) tmem_dealloc(tmem_base, Cfg::kTmemCols);
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

template <int NT>
cudaError_t launch_f4(const GemmF4Plan& p, int* d_err, cudaStream_t s) {
  F4KArgs a;
  a.a_mode = p.a_mode;
  a.T = p.T;
  a.out = p.out;
  a.sw0 = p.sw0;
  a.sw1 = p.sw1;
  a.sx = p.sx;
  a.err = d_err;
  return launch_k(k_gemm_fp4<NT>, dim3(p.out.grid), dim3(kF4Threads), F4Cfg<NT>::kSmem, s, p.tc0, p.tc1, p.ts0,
                  p.ts1, p.tb, a);
}

}  // namespace

size_t gemm_fp4_partial_bytes(int T, int N, int K, int a_mode) {
  GemmOut o;
  partition_f4(T, N, K, a_mode, &o);
  return (size_t)o.n_tiles * o.max_slots * ((T + 31) / 32 * 32) * kTileM * sizeof(float);
}

bool gemm_fp4_plan(GemmF4Plan* p, int a_mode, const dlm_nvfp4_matrix& w0, const dlm_nvfp4_matrix* w1,
                   const __half* xq, int x_rows, const float* sx, int T, int N, int K, float* partial, char* err,
                   size_t errlen) {
  memset(p, 0, sizeof(*p));
  const int nt = T <= 32 ? 32 : 64;
  if (T < 1 || T > kMaxF4Tokens || N < 1 || K < kF4K || K % kF4K != 0 || x_rows < nt ||
      (a_mode != A_KMAJOR && a_mode != A_PAIR) || (a_mode == A_PAIR && !w1) || !w0.codes || !w0.scales ||
      (w1 && (!w1->codes || !w1->scales)) || !xq || !sx) {
    snprintf(err, errlen, "nvfp4 gemm: unsupported arguments T=%d N=%d K=%d (K must be a multiple of %d, T <= %d)",
             T, N, K, kF4K, kMaxF4Tokens);
    return false;
  }
  p->a_mode = a_mode;
  p->T = T;
  p->N = N;
  p->K = K;
  p->nt = nt;
  p->sw0 = w0.tensor_scale;
  p->sw1 = w1 ? w1->tensor_scale : w0.tensor_scale;
  p->sx = sx;
  partition_f4(T, N, K, a_mode, &p->out);
  p->out.partial = partial;
  if ((unsigned long long)p->out.units * (unsigned long long)p->out.grid >= (1ull << 32)) {
    snprintf(err, errlen, "gemm: %ld units exceed the 32-bit partition arithmetic", p->out.units);
    return false;
  }
  p->partial_bytes = gemm_fp4_partial_bytes(T, N, K, a_mode);
  const uint32_t rows = (a_mode == A_PAIR) ? 64 : kTileM;
  bool ok = encode_2d(&p->tc0, CU_TENSOR_MAP_DATA_TYPE_UINT8, w0.codes, (uint64_t)K / 2, N, (uint64_t)K / 2, 128,
                      rows, CU_TENSOR_MAP_SWIZZLE_128B, err, errlen) &&
            encode_2d(&p->ts0, CU_TENSOR_MAP_DATA_TYPE_UINT8, w0.scales, (uint64_t)K / 16, N, (uint64_t)K / 16, 16,
                      rows, CU_TENSOR_MAP_SWIZZLE_NONE, err, errlen);
  if (ok && a_mode == A_PAIR) {
    ok = encode_2d(&p->tc1, CU_TENSOR_MAP_DATA_TYPE_UINT8, w1->codes, (uint64_t)K / 2, N, (uint64_t)K / 2, 128,
                   rows, CU_TENSOR_MAP_SWIZZLE_128B, err, errlen) &&
         encode_2d(&p->ts1, CU_TENSOR_MAP_DATA_TYPE_UINT8, w1->scales, (uint64_t)K / 16, N, (uint64_t)K / 16, 16,
                   rows, CU_TENSOR_MAP_SWIZZLE_NONE, err, errlen);
  } else {
    p->tc1 = p->tc0;
    p->ts1 = p->ts0;
  }
  ok = ok && encode_2d(&p->tb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xq, K, nt, (uint64_t)K * 2, 64, nt,
                       CU_TENSOR_MAP_SWIZZLE_128B, err, errlen);
  return ok;
}

cudaError_t gemm_fp4_launch(const GemmF4Plan& p, int* d_err, cudaStream_t s) {
  return p.nt == 32 ? launch_f4<32>(p, d_err, s) : launch_f4<64>(p, d_err, s);
}

int gemm_fp4_init_attributes() {
  static bool done = false;
  if (done) return 0;
  cudaError_t e = cudaFuncSetAttribute(k_gemm_fp4<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, F4Cfg<32>::kSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_fp4<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, F4Cfg<64>::kSmem);
  if (e == cudaSuccess) done = true;
  return (int)e;
}

}  // namespace dlm

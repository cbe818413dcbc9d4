// dlm_gemm.cu -- weight-streaming GEMM y[T][N] = x[T][K] W[N][K]^T for the dense
// projections of a denoising round (M = block size), on the sm_100a tensor cores.
//
// bs=1 rounds are bound by the HBM stream of the weights, so the kernel is shaped around
// that stream ("swap AB"): the weights are the 128-row A operand of tcgen05.mma, the
// block's tokens are the N = T operand, and the fp32 accumulator lives in TMEM.
//   * One warp issues TMA (cp.async.bulk.tensor, 128-byte swizzle) loads of the weight
//     tile and the activation tile of each k-block into an S-stage ring in shared memory.
//   * One thread issues the MMAs (4 x K=16 per k-block) and commits each stage back to
//     the producer; at the end of a tile it commits the accumulator to the epilogue.
//   * Four epilogue warps read the accumulator out of TMEM (tcgen05.ld) and store fp32
//     partial sums; two TMEM accumulators let the next tile's MMAs overlap the epilogue.
//   * Work is split stream-K: the (tile, k-block) units of the whole GEMM are cut into
//     `grid` equal contiguous ranges, one per SM, so every SM streams the same number of
//     weight bytes whatever the tile count.  A tile covered by several CTAs leaves one
//     partial per CTA ("slot"); the consumer sums the slots in a fixed order.
// No TMA multicast is used anywhere.
#include <cstdio>
#include <cstring>

#include "dlm_device.cuh"
#include "dlm_internal.h"

namespace dlm {

bool g_pdl = true;

template <int NT>
struct GemmCfg {
  static constexpr int kABytes = kTileM * kTileK * 2;          // 16 KB
  static constexpr int kBBytes = NT * kTileK * 2;              // NT rows of 128 B
  static constexpr int kStageBytes = kABytes + kBBytes;        // multiple of 1024
  static constexpr int kStages = NT <= 64 ? 8 : (NT <= 128 ? 6 : 4);
  static constexpr int kXchBytes = 128 * 33 * 4;                // epilogue row exchange
  static constexpr int kSmem = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/ + kXchBytes;
  static constexpr int kTmemCols = (2 * NT < 32) ? 32 : 2 * NT;  // power of two for NT >= 16
};

struct GemmKArgs {
  int a_mode;
  int T;
  int N;       // valid output rows (features)
  int lo_col;  // 0, or the MMA column where the low halves of split activations start
  GemmOut out;
  EpiArgs epi;
  int* err;
};

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

struct EpiSync {
  __device__ __forceinline__ void operator()() const { epi_sync(); }
};

// 192 threads: warp 0 = TMA producer (and TMEM allocator), warp 1 = MMA issuer,
// warps 2..5 = epilogue (TMEM lane quarter = warp % 4).
template <int NT>
__global__ void __launch_bounds__(192, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap ta1,
          const __grid_constant__ CUtensorMap tb, GemmKArgs args) {
  using Cfg = GemmCfg<NT>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + S * Cfg::kStageBytes);
  uint64_t* full = bars;            // [S]
  uint64_t* empty = bars + S;       // [S]
  uint64_t* acc_full = bars + 2 * S;   // [2]
  uint64_t* acc_empty = bars + 2 * S + 2;  // [2]
  uint64_t* mma_done = bars + 2 * S + 4;   // [1]
  uint32_t* tmem_holder = (uint32_t*)(bars + 2 * S + 5);
  int* last_flag = (int*)(bars + 2 * S + 6);
  float(*xch)[33] = reinterpret_cast<float(*)[33]>(smem + S * Cfg::kStageBytes + 256);

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
    tmem_alloc(tmem_holder, Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&ta0);
    if (args.a_mode == A_PAIR || args.a_mode == A_MNMAJOR) prefetch_tmap(&ta1);
    prefetch_tmap(&tb);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  if (warp != 0) pdl_wait();  // the producer waits after requesting its first weight tiles

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    uint32_t armed_parity[8];
    bool armed[8];
    for (int i = 0; i < S; ++i) armed[i] = false;
    auto load_a = [&](long u, int st) {
      const int tile = (int)(u / o.n_kb), kb = (int)(u % o.n_kb);
      uint8_t* sa = smem + st * Cfg::kStageBytes;
      if (args.a_mode == A_KMAJOR) {
        tma_load_2d(sa, &ta0, &full[st], kb * kTileK, tile * kTileM);
      } else if (args.a_mode == A_PAIR) {
        tma_load_2d(sa, &ta0, &full[st], kb * kTileK, tile * 64);
        tma_load_2d(sa + Cfg::kABytes / 2, &ta1, &full[st], kb * kTileK, tile * 64);
      } else {  // A^T stored [K][N]: two 64-wide column boxes of 64 K-rows
        tma_load_2d(sa, &ta0, &full[st], tile * kTileM, kb * kTileK);
        tma_load_2d(sa + Cfg::kABytes / 2, &ta0, &full[st], tile * kTileM + 64, kb * kTileK);
      }
    };
    auto load_b = [&](long u, int st) {
      const int kb = (int)(u % o.n_kb);
      tma_load_2d(smem + st * Cfg::kStageBytes + Cfg::kABytes, &tb, &full[st], kb * kTileK, 0);
    };
    // The weights do not depend on the previous kernel: the first S stages of them are
    // requested before waiting for it, the activations only after.
    const long n_pre = (u_end - u_begin) < S ? (u_end - u_begin) : S;
    for (long i = 0; i < n_pre; ++i) {
      mbar_arrive_expect_tx(&full[i], Cfg::kStageBytes);
      armed[i] = true;
      armed_parity[i] = 0;
      load_a(u_begin + i, (int)i);
    }
    pdl_wait();
    for (long i = 0; i < n_pre; ++i) load_b(u_begin + i, (int)i);
    int stage = (int)(n_pre % S);
    uint32_t phase = (n_pre == S) ? 1u : 0u;
    bool ok = true;
    for (long u = u_begin + n_pre; u < u_end && ok; ++u) {
      if (!mbar_wait(&empty[stage], phase ^ 1, args.err)) { ok = false; break; }
      mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
      armed[stage] = true;
      armed_parity[stage] = phase;
      load_a(u, stage);
      load_b(u, stage);
      if (++stage == S) { stage = 0; phase ^= 1; }
    }
    pdl_trigger();  // all loads issued: the next kernel may start its prologue
    // never leave the CTA with copies in flight: wait (bounded) for every armed stage
    for (int i = 0; i < S; ++i)
      if (armed[i]) mbar_wait(&full[i], armed_parity[i], args.err);
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp runs the loop and waits (outcomes made
    // warp-uniform); one elected lane issues the MMAs and the commits
    const uint32_t idesc = idesc_bf16(128, NT, args.a_mode == A_MNMAJOR, false);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    long u = u_begin;
    while (u < u_end && ok) {
      const int tile = (int)(u / o.n_kb);
      const long seg_end = ((long)tile + 1) * o.n_kb < u_end ? ((long)tile + 1) * o.n_kb : u_end;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_empty[acc], acc_phase ^ 1, args.err))) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * NT;
      for (long uu = u; uu < seg_end; ++uu) {
        if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, args.err))) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * Cfg::kStageBytes);
        const uint32_t sb = sa + Cfg::kABytes;
        // K step k: +32 B (K-major A and B) or +2048 B (MN-major A: 16 rows of 128 B)
        const uint64_t ad = (args.a_mode == A_MNMAJOR) ? sw128_desc(sa, Cfg::kABytes / 2, 1024)
                                                        : sw128_desc(sa, 16, 1024);
        const uint32_t astep = (args.a_mode == A_MNMAJOR) ? 128u : 2u;
        const uint64_t bd = sw128_desc(sb, 16, 1024);
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < kTileK / 16; ++k)
            mma_bf16(d_tmem, ad + astep * k, bd + 2 * k, idesc, (uu > u || k > 0) ? 1u : 0u);
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
    // all MMAs of the issuing lane complete before TMEM is released
    if (elect_one()) {
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, args.err);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> partial sums / finished tiles
    const int quarter = warp % 4;
    const int row = quarter * 32 + lane;  // tile row = TMEM lane
    const int et = threadIdx.x - 64;      // 0 .. 127
    const EpiArgs& e = args.epi;
    const int L = (e.op == EPI_QKV) ? (e.pos0_dev ? *e.pos0_dev + e.pos_off : e.pos0) : 0;
    const int ncb = (args.T + 31) / 32;
    int acc = 0;
    uint32_t acc_phase = 0;
    long u = u_begin;
    const int TP = ncb * 32;  // tokens padded to 32 in the partial layout
    float v[32];
    auto load_block = [&](uint32_t taddr, int cb) {
      tmem_ld32(taddr + cb * 32, v);
      if (args.lo_col) {
        // split activation x = hi + lo: the two column sets add up
        float w[32];
        tmem_ld32(taddr + args.lo_col + cb * 32, w);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += w[j];
      }
    };
    while (u < u_end) {
      const int tile = (int)(u / o.n_kb);
      const long seg_end = ((long)tile + 1) * o.n_kb < u_end ? ((long)tile + 1) * o.n_kb : u_end;
      // one thread polls the accumulator barrier; the named barrier hands the outcome to
      // all 128 epilogue threads so they leave (on a timeout) or go on together
      if (et == 0) *last_flag = mbar_wait(&acc_full[acc], acc_phase, args.err) ? 1 : 0;
      epi_sync();
      const bool got = *last_flag != 0;
      epi_sync();
      if (!got) break;
      tc_fence_after();
      const int lo_c = cta_of_unit((long)tile * o.n_kb, o.units, o.grid);
      const int hi_c = cta_of_unit((long)(tile + 1) * o.n_kb - 1, o.units, o.grid);
      const int nslots = hi_c - lo_c + 1, slot = c - lo_c;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * NT;
      // partials: [tile][slot][TP][128] fp32 (token-major; a warp's rows are contiguous)
      float* const tile_part = o.partial + (size_t)tile * o.max_slots * kTileM * TP + row;
      bool finisher = true;
      if (nslots > 1 || e.op == EPI_PARTIAL) {
        float* dst = tile_part + (size_t)slot * kTileM * TP;
        float* const blk = dst - row;  // the (tile, slot) block: [TP][128] fp32, contiguous
        if (e.op == EPI_PARTIAL && ncb == 1 && ((uintptr_t)blk & 15) == 0) {
          // 32 tokens: the 16 KB block goes out through shared memory as one bulk copy
          load_block(taddr, 0);
          tc_fence_before();
          mbar_arrive(&acc_empty[acc]);  // the accumulator can take the next tile now
          if (et == 0) bulk_wait_read_all();  // the previous segment's copy has left the buffer
          epi_sync();
          float* const stg = &xch[0][0];  // [32][128] fp32 inside the exchange buffer
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[j * kTileM + row] = v[j];
          fence_async_shared();
          epi_sync();
          if (et == 0) {
            bulk_store_s2g(blk, smem_u32(stg), 32 * kTileM * 4);
            bulk_commit();
          }
        } else {
#pragma unroll 1
          for (int cb = 0; cb < ncb; ++cb) {
            load_block(taddr, cb);
#pragma unroll
            for (int j = 0; j < 32; ++j) dst[(size_t)(cb * 32 + j) * kTileM] = v[j];
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[acc]);  // the accumulator can take the next tile now
        }
        if (e.op == EPI_PARTIAL) {
          finisher = false;
        } else {
          __threadfence();
          epi_sync();
          if (et == 0) *last_flag = (atomicAdd(&e.tile_cnt[tile], 1) == nslots - 1) ? 1 : 0;
          epi_sync();
          finisher = *last_flag != 0;
          epi_sync();  // the flag is rewritten by the next segment's wait
          if (finisher) __threadfence();
        }
      }
      if (finisher) {
#pragma unroll 1
        for (int cb = 0; cb < ncb; ++cb) {
          if (nslots == 1) {
            load_block(taddr, cb);
          } else {
            sum_slots32(o, tile, row, cb * 32, TP, nslots, v);
          }
          apply_epi(args.epi, args.N, args.T, tile, row, cb * 32, v, xch, L, EpiSync());
        }
        if (nslots == 1) {
          tc_fence_before();
          mbar_arrive(&acc_empty[acc]);
        } else if (et == 0) {
          e.tile_cnt[tile] = 0;  // ready for the next GEMM
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      u = seg_end;
    }
    if (et == 0) bulk_wait_all();  // partial sums written before the CTA ends
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, Cfg::kTmemCols);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_encodeTiled)p;
  }
  return fn;
}

bool encode_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, char* err,
                    size_t errlen) {
  return encode_tmap_2d_swizzle(map, base, inner, outer, row_bytes, box_inner, box_outer, 128, err, errlen);
}

bool encode_tmap_2d_swizzle(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                            uint32_t box_inner, uint32_t box_outer, int swizzle_bytes, char* err, size_t errlen) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled entry point unavailable");
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : (swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE);
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled failed (%d): dims %llu x %llu box %u x %u", (int)r,
             (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
    return false;
  }
  return true;
}

static int pad_nt(int T) {
  if (T <= 32) return 32;
  if (T <= 64) return 64;
  if (T <= 128) return 128;
  return 256;
}

static void partition(int T, int N, int K, int a_mode, GemmOut* o) {
  const int rows_per_tile = (a_mode == A_PAIR) ? 64 : kTileM;
  o->T = T;
  o->n_tiles = (N + rows_per_tile - 1) / rows_per_tile;
  o->n_kb = (K + kTileK - 1) / kTileK;
  o->units = (long)o->n_tiles * o->n_kb;
  int grid = kSMs;
  if (o->units < grid) grid = (int)o->units;
  o->grid = grid;
  int ms = 1;
  for (int t = 0; t < o->n_tiles; ++t) {
    int lo = cta_of_unit((long)t * o->n_kb, o->units, grid);
    int hi = cta_of_unit((long)(t + 1) * o->n_kb - 1, o->units, grid);
    if (hi - lo + 1 > ms) ms = hi - lo + 1;
  }
  o->max_slots = ms;
}

size_t gemm_partial_bytes(int T, int N, int K, int a_mode) {
  GemmOut o;
  partition(T, N, K, a_mode, &o);
  return (size_t)o.n_tiles * o.max_slots * ((T + 31) / 32 * 32) * kTileM * sizeof(float);
}

int split_pad(int T) { return T <= 32 ? 32 : (T <= 64 ? 64 : 128); }

bool gemm_plan(GemmPlan* p, int a_mode, const void* a0, const void* a1, const void* x, int T, int N,
               int K, float* partial, char* err, size_t errlen, bool split) {
  memset(p, 0, sizeof(*p));
  if (T < 1 || T > (split ? kMaxSplitTokens : kMaxTokens) || N < 1 || K < kTileK || K % 8 != 0) {
    snprintf(err, errlen, "gemm: unsupported shape T=%d N=%d K=%d split=%d", T, N, K, (int)split);
    return false;
  }
  p->a_mode = a_mode;
  p->a0 = a0;
  p->a1 = a1;
  p->x = x;
  p->N = N;
  p->K = K;
  p->T = T;
  p->nt = split ? 2 * split_pad(T) : pad_nt(T);
  p->lo_col = split ? split_pad(T) : 0;
  partition(T, N, K, a_mode, &p->out);
  p->out.partial = partial;
  if ((unsigned long long)p->out.units * (unsigned long long)p->out.grid >= (1ull << 32)) {
    snprintf(err, errlen, "gemm: %ld units exceed the 32-bit partition arithmetic", p->out.units);
    return false;
  }
  p->partial_bytes = gemm_partial_bytes(T, N, K, a_mode);
  bool ok = true;
  if (a_mode == A_KMAJOR) {
    ok = encode_tmap_2d(&p->ta0, a0, K, N, (uint64_t)K * 2, kTileK, kTileM, err, errlen);
    p->ta1 = p->ta0;
  } else if (a_mode == A_PAIR) {
    ok = encode_tmap_2d(&p->ta0, a0, K, N, (uint64_t)K * 2, kTileK, 64, err, errlen) &&
         encode_tmap_2d(&p->ta1, a1, K, N, (uint64_t)K * 2, kTileK, 64, err, errlen);
  } else {
    // A^T stored [K][N] row-major: inner dimension N, boxes of 64 (N) x 64 (K rows)
    ok = encode_tmap_2d(&p->ta0, a0, N, K, (uint64_t)N * 2, 64, kTileK, err, errlen);
    p->ta1 = p->ta0;
  }
  // split activations: rows [0, T) high halves, rows [pad, pad + T) low halves
  ok = ok && encode_tmap_2d(&p->tb, x, K, split ? p->nt : T, (uint64_t)K * 2, kTileK, p->nt, err, errlen);
  return ok;
}

template <int NT>
static cudaError_t launch_nt(const GemmPlan& p, int* d_err, cudaStream_t s) {
  GemmKArgs a;
  a.a_mode = p.a_mode;
  a.T = p.T;
  a.N = p.N;
  a.lo_col = p.lo_col;
  a.out = p.out;
  a.epi = p.epi;
  a.err = d_err;
  return launch_k(k_gemm_tc<NT>, dim3(p.out.grid), dim3(192), GemmCfg<NT>::kSmem, s, p.ta0, p.ta1, p.tb, a);
}

template <int NT>
static cudaError_t set_smem_attr() {
  return cudaFuncSetAttribute(k_gemm_tc<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<NT>::kSmem);
}

// Sets the dynamic shared-memory limits of every GEMM instantiation once per device (must
// happen outside stream capture).
int gemm_init_attributes() {
  static PerDeviceOnce once;
  return once_on_current_device(once, [] {
    cudaError_t e = set_smem_attr<32>();
    if (e == cudaSuccess) e = set_smem_attr<64>();
    if (e == cudaSuccess) e = set_smem_attr<128>();
    if (e == cudaSuccess) e = set_smem_attr<256>();
    return (int)e;
  });
}

cudaError_t gemm_launch(const GemmPlan& p, int* d_err, cudaStream_t s) {
  switch (p.nt) {
    case 32: return launch_nt<32>(p, d_err, s);
    case 64: return launch_nt<64>(p, d_err, s);
    case 128: return launch_nt<128>(p, d_err, s);
    default: return launch_nt<256>(p, d_err, s);
  }
}

}  // namespace dlm

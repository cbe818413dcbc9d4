// dlm_device.cuh -- device-side helpers shared by the sm_100a kernels: PTX wrappers for
// mbarriers, TMA bulk-tensor loads, tcgen05 (TMEM allocation, MMA, commit, loads) and
// bounded waits.  Every wait gives up after a fixed number of polls and records an
// error code in device memory instead of hanging the GPU.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dlm_internal.h"

namespace dlm {

// ---------------------------------------------------------------- misc
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ __nv_bfloat16 f2bf(float x) { return __float2bfloat16_rn(x); }

// Stores v as a split bf16 pair: the high half at p[0] and, when lo_off != 0, the
// rounding remainder at p[lo_off] (hi + lo carries about 16 significant bits).
__device__ __forceinline__ void store_split(__nv_bfloat16* p, long lo_off, float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  p[0] = h;
  if (lo_off) p[lo_off] = __float2bfloat16_rn(v - __bfloat162float(h));
}

// ---------------------------------------------------------------- programmatic dependent launch
// Every kernel of a round lets the next kernel in the stream launch as soon as all of its
// own CTAs are running (pdl_trigger at entry), and waits for the previous kernel to
// complete and flush (pdl_wait) before it reads or writes any mutable global memory.
// Only constant data (weights) may be touched before pdl_wait.  Both are no-ops for a
// kernel launched without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Records the first error code seen by any thread (0 = no error).
__device__ __forceinline__ void set_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns false (and
// records DLM_ETIMEOUT) after about kWaitPolls polls, i.e. well over a second.
constexpr uint32_t kWaitPolls = 1u << 24;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err) {
  for (uint32_t i = 0; i < kWaitPolls; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (i >= 16) __nanosleep(i < 1024 ? 32 : 256);
  }
  set_error(err, DLM_ETIMEOUT);
  return false;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// The same load with an L2 eviction-priority policy (see l2_policy_*).
__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x,
                                                 int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
// L2 policies: keep lines that will be read again soon / let lines read for the last time go.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- bulk copies to global
// Shared-memory writes of this thread visible to the async proxy (a bulk copy reading them).
__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Bulk copy of `bytes` (a multiple of 16) from shared memory to global memory, both 16-byte
// aligned, in the issuing thread's current bulk group.
__device__ __forceinline__ void bulk_store_s2g(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// This thread's bulk copies have read their shared-memory sources / have completed.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One lane of a fully active warp (the same lane on every call: the lowest).  An MMA loop run
// by the whole warp, with the issue and commit under elect_one(), issues faster than the same
// loop run by a single thread (its values stay warp-uniform).
__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.u32 %0, 1, 0, e;\n\t}" : "=r"(p));
  return p != 0;
}

// Arrives on the mbarrier once all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor (tcgen05 format, version 1) for a 128-byte-swizzled
// operand.  For K-major tiles: rows of 128 B, 8-row groups 1024 B apart (SBO).  For
// MN-major tiles: `lbo` is the byte distance between 64-element MN atoms and SBO the
// distance between 8-row K groups.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFF);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;   // descriptor version for sm_100
  d |= uint64_t(2) << 61;   // SWIZZLE_128B
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 D, M = 128 (or 64), N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                       // D format fp32
         | (1u << 7)                     // A bf16
         | (1u << 10)                    // B bf16
         | (uint32_t(a_mn_major) << 15)  // A major
         | (uint32_t(b_mn_major) << 16)  // B major
         | (uint32_t(n >> 3) << 17)      // N / 8
         | (uint32_t(m >> 4) << 24);     // M / 16
}

// Token scales of an NVFP4 GEMM input (K elements per row): one plane per group of 32 tokens,
// [group][64-element block][token % 32][16 B], byte k of a row's 16 the scale of its
// 16-element group 4 b + k (4 of the 16 bytes used), so that a stage's four blocks of one
// group are 2 KB of contiguous tcgen05.cp sources.  b16 = index of the 16-element block.
__host__ __device__ __forceinline__ size_t tok_scale_index(int t, int b16, int K) {
  return ((size_t)(t >> 5) * (size_t)(K / 64) + (size_t)(b16 >> 2)) * 512 + (size_t)(t & 31) * 16 + (size_t)(b16 & 3);
}

// ---------------------------------------------------------------- block-scaled FP4 MMA
// Shared-memory descriptor of a 32-row x 16-byte block without swizzle (the tcgen05.cp
// source): core matrices of 8 rows x 16 bytes, 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFF);
  d |= uint64_t(128 >> 4) << 16;  // leading byte offset (one core matrix along K: unused)
  d |= uint64_t(128 >> 4) << 32;  // stride byte offset: next 8 rows
  d |= uint64_t(1) << 46;         // descriptor version for sm_100
  return d;                       // layout type 0: no swizzle
}

__device__ __forceinline__ void tmem_cp_32x128(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with e2m1 operands and e4m3 scales per 16 elements.
__device__ __forceinline__ void mma_nvf4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

// Instruction descriptor of kind::mxf4nvf4: A and B e2m1 (format 1), K-major, e4m3 scales,
// M = m, N = n, K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(int m, int n) {
  return (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}


// Instruction descriptor of kind::f16 with f16 A/B, fp32 D, M = m, N = n.
__host__ __device__ constexpr uint32_t idesc_f16(int m, int n, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                       // D format fp32
         | (0u << 7)                     // A f16
         | (0u << 10)                    // B f16
         | (uint32_t(a_mn_major) << 15)
         | (uint32_t(b_mn_major) << 16)
         | (uint32_t(n >> 3) << 17)
         | (uint32_t(m >> 4) << 24);
}

// ---------------------------------------------------------------- stream-K partition
// The (tile, k-block) units of a GEMM are cut into `grid` contiguous ranges; CTA c owns
// units [unit_begin(c), unit_begin(c + 1)).
// 32-bit arithmetic (the planners keep units * grid below 2^32; a 64-bit division costs
// about a hundred instructions on the critical path of every finishing thread).
__host__ __device__ __forceinline__ long unit_begin(int c, long units, int grid) {
  return (long)((uint32_t)c * (uint32_t)units / (uint32_t)grid);
}
// Largest CTA index c with unit_begin(c) <= u.
__host__ __device__ __forceinline__ int cta_of_unit(long u, long units, int grid) {
  int c = (int)((uint32_t)u * (uint32_t)grid / (uint32_t)units);
  if (c >= grid) c = grid - 1;
  while (c + 1 < grid && unit_begin(c + 1, units, grid) <= u) ++c;
  while (c > 0 && unit_begin(c, units, grid) > u) --c;
  return c;
}

// Partial sums: [tile][slot][TP][128] fp32 with TP = T rounded up to 32.  sum_slots32 adds
// the slots of (tile, row) for tokens t0 .. t0+31 in slot order, NB slots of 32 independent
// loads in flight at a time (L2 reads: the partials were written by other SMs).
template <int NB = 2>
__device__ __forceinline__ void sum_slots32(const GemmOut& o, int tile, int row, int t0, int TP, int nslots,
                                            float (&v)[32]) {
  const float* base = o.partial + (size_t)tile * o.max_slots * kTileM * TP + (size_t)t0 * kTileM + row;
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = 0.f;
  for (int sl = 0; sl < nslots; sl += NB) {
    float x[NB][32];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float* a = base + (size_t)(sl + b) * kTileM * TP;
      const bool ok = sl + b < nslots;
#pragma unroll
      for (int j = 0; j < 32; ++j) x[b][j] = (ok && t0 + j < o.T) ? __ldcg(a + (size_t)j * kTileM) : 0.f;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += x[b][j];  // slot order
    }
  }
}

__device__ __forceinline__ int tile_slots(const GemmOut& o, int tile) {
  return cta_of_unit((long)(tile + 1) * o.n_kb - 1, o.units, o.grid) - cta_of_unit((long)tile * o.n_kb, o.units, o.grid) + 1;
}

// Applies the epilogue op to one block of (up to) 32 tokens of a finished tile.  Runs on the
// 128 threads of which `row` is this thread's tile row and v[j] its value for token t0 + j;
// `sync` synchronizes those 128 threads.  N = valid output features, T = tokens, L = the
// position of token 0.
template <class Sync>
__device__ __forceinline__ void apply_epi(const EpiArgs& e, int N, int T, int tile, int row, int t0,
                                          const float (&v)[32], float (*xch)[33], int L, Sync sync) {
  const int nt = (T - t0) < 32 ? (T - t0) : 32;
  if (e.op == EPI_STORE) {
    const int n = tile * kTileM + row;
    if (n < N) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nt) e.out[(size_t)(t0 + j) * e.ld + n] = (e.scale != 0.f) ? v[j] * e.scale : v[j];
    }
  } else if (e.op == EPI_RESID || e.op == EPI_EMBED) {
    const int n = tile * kTileM + row;
    const bool ok = n < N;
    // all loads first (independent, in flight together), then the stores
    float base[32];
    if (e.op == EPI_RESID) {
#pragma unroll
      for (int j = 0; j < 32; ++j) base[j] = (ok && j < nt) ? e.h[(size_t)(t0 + j) * N + n] : 0.f;
    } else {
      int tok[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) tok[j] = (j < nt) ? e.tokens[t0 + j] : 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) base[j] = (ok && j < nt) ? bf2f(e.embed[(size_t)tok[j] * N + n]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float hn = 0.f;
      if (ok && j < nt) {
        hn = base[j] + v[j];
        e.h[(size_t)(t0 + j) * N + n] = hn;
      }
      xch[row][j] = hn * hn;
    }
    sync();
    if (row < nt) {
      float ss = 0.f;
      for (int r = 0; r < kTileM; ++r) ss += xch[r][row];
      e.ss[(size_t)tile * T + t0 + row] = ss;
    }
    sync();
  } else if (e.op == EPI_SILU) {
#pragma unroll
    for (int j = 0; j < 32; ++j) xch[row][j] = v[j];
    sync();
    const int f = tile * 64 + row;
    if (row < 64 && f < N) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < nt) {
          const float g = xch[row][j], u = xch[row + 64][j];
          const float silu = g / (1.0f + expf(-g));
          store_split(e.act + (size_t)(t0 + j) * N + f, e.act_lo, silu * u);
        }
      }
    }
    sync();
  } else if (e.op == EPI_QKV) {
#pragma unroll
    for (int j = 0; j < 32; ++j) xch[row][j] = v[j];
    sync();
    const int n = tile * kTileM + row;
    const int hd = e.hd, half = hd / 2;
    const int hh = n / hd, jj = n % hd;
    if (n < N) {
      const int partner = (jj < half) ? row + half : row - half;
      const bool rope = hh < e.Hq + e.Hkv;
      const float2* tab = e.rope_tab + (jj % half);  // (cos, sin) at [position][jj % half]
      __nv_bfloat16* dst;
      size_t stride_t;
      if (hh < e.Hq) {
        dst = e.q + (size_t)hh * hd + jj;
        stride_t = (size_t)e.Hq * hd;
      } else if (hh < e.Hq + e.Hkv) {
        dst = e.kc + ((size_t)(hh - e.Hq) * e.max_ctx + L) * hd + jj;
        stride_t = hd;
      } else {
        dst = e.vc + ((size_t)(hh - e.Hq - e.Hkv) * e.max_ctx + L) * hd + jj;
        stride_t = hd;
      }
      float2 cs[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) cs[j] = (rope && j < nt) ? tab[(size_t)(L + t0 + j) * half] : make_float2(1.f, 0.f);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < nt) {
          float out = xch[row][j];
          if (rope) {
            const float pv = xch[partner][j];
            out = (jj < half) ? out * cs[j].x - pv * cs[j].y : pv * cs[j].y + out * cs[j].x;
          }
          dst[(size_t)(t0 + j) * stride_t] = f2bf(out);
        }
      }
    }
    sync();
  }
}

// ---------------------------------------------------------------- NVFP4 number formats
// e2m1 code of r (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6; ties to the even code; sign in bit 3).
__device__ __forceinline__ uint8_t e2m1_rne(float r) {
  const float a = fabsf(r);
  uint8_t c;
  if (a <= 0.25f) c = 0;
  else if (a < 0.75f) c = 1;
  else if (a <= 1.25f) c = 2;
  else if (a < 1.75f) c = 3;
  else if (a <= 2.5f) c = 4;
  else if (a < 3.5f) c = 5;
  else if (a <= 5.0f) c = 6;
  else c = 7;
  return (uint8_t)(c | ((r < 0.f) ? 8 : 0));
}

// Value of an e2m1 code (bit 3 = sign).
__device__ __forceinline__ float e2m1_value_dev(uint8_t c) {
  const int m = c & 7;
  const float mag = (m < 4) ? 0.5f * m : (m < 6 ? (float)(m - 2) : (m == 6 ? 4.0f : 6.0f));
  return (c & 8) ? -mag : mag;
}

// Value of an e4m3 byte (sign bit ignored: scales are non-negative).
__device__ __forceinline__ float e4m3_value_dev(uint8_t b) {
  int E = (b >> 3) & 15, m = b & 7;
  if (E == 0) return ldexpf((float)m, -9);
  return ldexpf(1.0f + m / 8.0f, E - 7);
}

// Rounds a non-negative fp32 value to e4m3 (RNE, saturating at 448); returns the bits.
__device__ __forceinline__ uint8_t e4m3_rne_bits(float x) {
  if (!(x > 0.f)) return 0;
  if (x >= 448.f) return 0x7E;
  int e;
  frexpf(x, &e);  // x = f 2^e, f in [0.5, 1)
  int qexp = e - 4;
  if (qexp < -9) qexp = -9;
  float q = ldexpf(1.0f, qexp);
  float r = rintf(x / q) * q;  // x / q exact (power of two), rintf: ties to even
  if (r > 448.f) r = 448.f;
  // encode r
  int e2;
  float f2 = frexpf(r, &e2);
  int E = e2 - 1 + 7;
  if (E <= 0) return (uint8_t)((int)rintf(r / ldexpf(1.0f, -9)) & 7);
  int mm = (int)rintf((f2 * 2.0f - 1.0f) * 8.0f);
  return (uint8_t)((E << 3) | mm);
}

// ---------------------------------------------------------------- warp reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace dlm

// dlm_lmhead.cu -- the LM head fused with the row statistics and the residual contraction,
// in one pass over the tied embedding E:
//   logits = x E^T (never stored), per row: max, lowest argmax, Z = sum e^(l - r),
//   A = sum e^(l - r) l for a reference r, and s = P E with P = softmax(logits) (or a
//   given P).
// ("QwenDLM-4B-ORL" model card, "The paper's evaluation pipeline": the LM head runs with
// fused row statistics; "ORL: diffusion LLMs get a learnable 'tokens per forward'", "What
// shipped": the previous round's distribution is fed back through the tied embedding.)
//
// Work split: vocabulary tiles of 128 rows, a contiguous range of tiles per cluster of two
// CTAs; CTA rank r owns the model-width half [r d/2, (r + 1) d/2).  Per tile:
//   L  partial logits over the CTA's half: tcgen05, A = E tile (K-major), B = x as a split
//      bf16 pair (N = 64: the high halves in TMEM columns 0..31, the low halves in 32..63,
//      added by the epilogue), so each E chunk is read once per MMA; double-buffered.
//   X  the two partial logit tiles are swapped through distributed shared memory (remote
//      stores + a remote mbarrier arrive with cluster-scope release), so both CTAs hold
//      the same full logits; they are read transposed ([token][vocab]) for the per-token
//      reductions.  Running reference r_t: the first tile's max, raised (and the
//      accumulators rescaled) only when a tile's max exceeds it by more than 8.
//   PE s^T[d][t] += E_tile^T P_tile: tcgen05 with A = the same E tile re-read (from L2) as
//      an MN-major operand and B = P written by the epilogue into shared memory as a split
//      bf16 pair; s stays in TMEM (one 128-row x 32-column accumulator per 128 features).
// The MMA warp issues L(i + 1) before PE(i) so the statistics of tile i overlap the next
// tile's weight stream.  A cluster leaves (r, Z, A, max, argmax) per token and its s half;
// k_lmf_combine merges the clusters in a fixed order.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "dlm_device.cuh"
#include "dlm_internal.h"

namespace dlm {

namespace {

constexpr int kLmT = 32;                // tokens (MMA N)
constexpr int kLmStages = 6;
constexpr int kLmStageBytes = 24576;    // E box 16 KB + x box 8 KB (L) / 2 E boxes + P box (PE)
constexpr int kLmPBytes = 16384;        // P tile: 64 rows (hi, lo) x 128 vocab, 2 swizzle atoms
constexpr int kLmXBytes = kLmT * 128 * 4;  // one partial-logit tile [32][128] fp32
constexpr int kLmMaxChunks = 12;        // d / 2 <= 1536 (TMEM: 128 + 12 x 32 columns)
constexpr int kLmMaxClusters = kSMs / 2;  // clusters of two CTAs (<= 80: five per merge chunk)
constexpr int kLmSCol = 128;            // TMEM column of the first s accumulator
constexpr float kLmRescale = 8.0f;      // raise the reference when a max exceeds it by this
constexpr int kLmSmem = kLmStages * kLmStageBytes + 2 * kLmPBytes + 3 * kLmXBytes + 1024 + 1024;
static_assert(kLmSmem <= 232448, "fused LM head shared memory");

struct LmfArgs {
  int V, d, T, mask_id;
  int x_hi_row, x_lo_row;  // rows of the split x where the high / low halves start
  int n_tiles, n_clu;
  int given;            // 1: P comes from memory (tp), s = P E without normalisation
  float* part_stats;    // [n_clu][32][4]: reference, Z, A, max
  int* part_arg;        // [n_clu][32]
  float* part_s;        // [n_clu][d][32]
  int* err;
  float s_scale;        // multiplies s (the NVFP4 E tensor scale; 1 for bf16 E)
  const float* sx;      // NVFP4: per-token scales of the quantized x
  float se;             // NVFP4: tensor scale of E
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_peer(uint32_t local_addr, uint32_t peer) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(peer));
  return r;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, int* err) {
  for (uint32_t i = 0; i < kWaitPolls; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
    if (i >= 16) __nanosleep(i < 1024 ? 32 : 256);
  }
  set_error(err, DLM_ETIMEOUT);
  return false;
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tmem_st32_f(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
      "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
      "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Barrier of the 128 epilogue threads that also returns whether any of them passed true.
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__host__ __device__ __forceinline__ int lm_tile_begin(int c, int n_tiles, int n_clu) {
  return (int)((long)c * n_tiles / n_clu);
}

// Offset of element (row, v) of the P tile (K-major B operand, 128-byte swizzle, two 64-wide
// atoms of 64 rows each).
__device__ __forceinline__ uint32_t p_offset(int row, int v) {
  const int atom = v >> 6, c = v & 63;
  return (uint32_t)(atom * 8192 + row * 128 + ((((c >> 3) ^ (row & 7)) << 4) | ((c & 7) << 1)));
}

__global__ void __launch_bounds__(192, 1)
k_lmhead_fused(const __grid_constant__ CUtensorMap tek, const __grid_constant__ CUtensorMap tem,
               const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tp, LmfArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;
  uint8_t* pbuf = smem + kLmStages * kLmStageBytes;                     // [2][16 KB]
  // mine: this CTA's own partial logits of the current tile (one buffer: every epilogue
  // thread has finished reading tile i, a barrier later, before any writes tile i + 1);
  // theirs: the peer's, written remotely and possibly one tile ahead (two buffers)
  float* mine = (float*)(pbuf + 2 * kLmPBytes);                         // [32][128]
  float* theirs = mine + kLmT * 128;                                    // [2][32][128]
  uint64_t* bars = (uint64_t*)(theirs + 2 * kLmT * 128);
  uint64_t* full = bars;                      // [S]
  uint64_t* empty = bars + kLmStages;         // [S]
  uint64_t* accl_full = bars + 2 * kLmStages; // [2]
  uint64_t* accl_empty = accl_full + 2;       // [2] (128 arrivals)
  uint64_t* p_ready = accl_empty + 2;         // [2] (4 arrivals)
  uint64_t* pe_done = p_ready + 2;            // [2]
  uint64_t* xfull = pe_done + 2;              // [2] (128 remote arrivals from the peer)
  uint64_t* mma_done = xfull + 2;
  uint32_t* tmem_holder = (uint32_t*)(mma_done + 1);
  int* flag = (int*)(mma_done + 2);
  float* fac = (float*)(mma_done + 3);        // [32] rescale factors of the current tile

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const int clu = blockIdx.x / 2;
  const int dh = a.d / 2, d0 = (int)rank * dh;
  const int KB = dh / 64, CH = dh / 128;
  const int tb = lm_tile_begin(clu, a.n_tiles, a.n_clu), te = lm_tile_begin(clu + 1, a.n_tiles, a.n_clu);
  const int nt = te - tb;

  if (warp == 1 && lane == 0) {
    for (int i = 0; i < kLmStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accl_full[i], 1);
      mbar_init(&accl_empty[i], 128);
      mbar_init(&p_ready[i], 4);
      mbar_init(&pe_done[i], 1);
      mbar_init(&xfull[i], 128);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tek);
    prefetch_tmap(&tem);
    prefetch_tmap(&tx);
    if (a.given) prefetch_tmap(&tp);
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_trigger();
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer: L(0), L(1), PE(0), L(2), PE(1), ..., PE(nt - 1)
    // E tiles are read twice (L from HBM, PE about two tiles later): the first read asks L2
    // to keep the lines, the second lets them go; x is read for every tile and kept.
    const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto next_stage = [&]() -> uint8_t* {
      if (!mbar_wait(&empty[stage], phase ^ 1, a.err)) { ok = false; return nullptr; }
      return ring + stage * kLmStageBytes;
    };
    auto advance = [&]() { if (++stage == kLmStages) { stage = 0; phase ^= 1; } };
    auto load_l = [&](int i) {
      const int tile = tb + i;
      for (int kb = 0; kb < KB && ok; ++kb) {
        uint8_t* st = next_stage();
        if (!ok) break;
        mbar_arrive_expect_tx(&full[stage], 16384 + 8192);
        tma_load_2d_hint(st, &tek, &full[stage], d0 + kb * 64, tile * 128, keep);
        // x: 32 rows of high halves, then 32 rows of low halves (a 64-row K-major B operand)
        tma_load_2d_hint(st + 16384, &tx, &full[stage], d0 + kb * 64, a.x_hi_row, keep);
        tma_load_2d_hint(st + 16384 + 4096, &tx, &full[stage], d0 + kb * 64, a.x_lo_row, keep);
        advance();
      }
    };
    auto load_pe = [&](int i) {
      const int tile = tb + i;
      for (int ch = 0; ch < CH && ok; ++ch)
        for (int vh = 0; vh < 2 && ok; ++vh) {
          uint8_t* st = next_stage();
          if (!ok) break;
          mbar_arrive_expect_tx(&full[stage], 16384 + (a.given ? 4096 : 0));
          tma_load_2d_hint(st, &tem, &full[stage], d0 + ch * 128, tile * 128 + vh * 64, drop);
          tma_load_2d_hint(st + 8192, &tem, &full[stage], d0 + ch * 128 + 64, tile * 128 + vh * 64, drop);
          if (a.given) tma_load_2d_hint(st + 16384, &tp, &full[stage], tile * 128 + vh * 64, 0, drop);
          advance();
        }
    };
    for (int i = 0; i < nt && ok; ++i) {
      load_l(i);
      if (i >= 1) load_pe(i - 1);
    }
    if (ok && nt > 0) load_pe(nt - 1);
    // no copies left in flight: wait for the stages still owned by the MMA warp
    for (int i = 0; i < kLmStages && ok; ++i) {
      if (!mbar_wait(&empty[stage], phase ^ 1, a.err)) break;
      advance();
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (same order as the producer).  The whole warp runs the loop
    // and waits; one elected lane issues the MMAs and commits (outcomes made warp-uniform).
    const uint32_t idesc_l = idesc_bf16(128, 2 * kLmT, false, false);
    const uint32_t idesc_pe = idesc_bf16(128, kLmT, true, false);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, a.err)) != 0;
    };
    auto mma_l = [&](int i) {
      const int b = i & 1;
      if (!wait_all(&accl_empty[b], ((i >> 1) & 1) ^ 1)) { ok = false; return; }
      tc_fence_after();
      const uint32_t dl = tmem + b * 2 * kLmT;
      for (int kb = 0; kb < KB; ++kb) {
        if (!wait_all(&full[stage], phase)) { ok = false; return; }
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + stage * kLmStageBytes);
        const uint64_t ad = sw128_desc(sa, 16, 1024), xd = sw128_desc(sa + 16384, 16, 1024);
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < 4; ++k)  // x box rows 0..31 = hi, 32..63 = lo -> D columns 0..63
            mma_bf16(dl, ad + 2 * k, xd + 2 * k, idesc_l, (kb | k) ? 1u : 0u);  // +32 B per k step
          mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kLmStages) { stage = 0; phase ^= 1; }
      }
      if (elect_one()) mma_commit(&accl_full[b]);
      __syncwarp();
    };
    auto mma_pe = [&](int i) {
      const int b = i & 1;
      if (!wait_all(&p_ready[b], (i >> 1) & 1)) { ok = false; return; }
      tc_fence_after();
      const uint64_t pd = sw128_desc(smem_u32(pbuf + b * kLmPBytes), 16, 1024);
      for (int ch = 0; ch < CH; ++ch) {
        const uint32_t ds = tmem + kLmSCol + ch * kLmT;
        for (int vh = 0; vh < 2; ++vh) {
          if (!wait_all(&full[stage], phase)) { ok = false; return; }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * kLmStageBytes);
          const uint64_t ad0 = sw128_desc(sa, 8192, 1024), gd = sw128_desc(sa + 16384, 16, 1024);
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t ad = ad0 + 128 * k;  // E^T: 16 vocab rows (2048 B) per step
              const bool first = (i == 0 && vh == 0 && k == 0);
              if (a.given) {
                mma_bf16(ds, ad, gd + 2 * k, idesc_pe, first ? 0u : 1u);
              } else {
#pragma unroll
                for (int h = 0; h < 2; ++h)  // P rows 0..31 = hi, 32..63 = lo (+4096 B)
                  mma_bf16(ds, ad, pd + (vh * 8192 + h * 4096 + k * 32) / 16, idesc_pe,
                           (first && h == 0) ? 0u : 1u);
              }
            }
            mma_commit(&empty[stage]);
          }
          __syncwarp();
          if (++stage == kLmStages) { stage = 0; phase ^= 1; }
        }
      }
      if (elect_one()) mma_commit(&pe_done[b]);
      __syncwarp();
    };
    for (int i = 0; i < nt && ok; ++i) {
      mma_l(i);
      if (ok && i >= 1) mma_pe(i - 1);
    }
    if (ok && nt > 0) mma_pe(nt - 1);
    if (elect_one()) {
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, a.err);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ---------------- epilogue: exchange, statistics, P, rescale, outputs
    const int et = threadIdx.x - 64;        // 0..127
    const int q = warp % 4, row = q * 32 + lane;   // TMEM lane of this thread
    const int tw = et / 32;                  // tokens 8 tw .. 8 tw + 7 in the transposed phase
    float ref[8], Z[8], A[8], mbest[8];
    int arg[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) { ref[j] = -INFINITY; Z[j] = 0.f; A[j] = 0.f; mbest[j] = -INFINITY; arg[j] = 0x7fffffff; }
    const uint32_t theirs_peer = map_peer(smem_u32(theirs), peer);
    const uint32_t xfull_peer = map_peer(smem_u32(xfull), peer);
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i) {
      const int b = i & 1, tile = tb + i;
      // 1. this CTA's partial logits of vocabulary row `row`, 32 tokens
      if (et == 0) *flag = mbar_wait(&accl_full[b], (i >> 1) & 1, a.err) ? 1 : 0;
      epi_bar();
      ok = *flag != 0;
      epi_bar();
      if (!ok) break;
      tc_fence_after();
      float lp[32];
      {
        float lo_[32];
        const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + b * 2 * kLmT;
        tmem_ld32(ta, lp);
        tmem_ld32(ta + kLmT, lo_);
#pragma unroll
        for (int t = 0; t < 32; ++t) lp[t] += lo_[t];
      }
      tc_fence_before();
      mbar_arrive(&accl_empty[b]);
      // 2. swap with the peer: own copy locally, the peer's copy by remote stores
      float* mb = mine;
      const uint32_t tpeer = theirs_peer + (uint32_t)(b * kLmT * 128 * 4);
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        mb[t * 128 + row] = lp[t];
        st_cluster_f32(tpeer + (uint32_t)((t * 128 + row) * 4), lp[t]);
      }
      mbar_arrive_remote(xfull_peer + b * 8);
      // every thread acquires the peer's tile itself; the barrier also publishes the local
      // partial writes to the transposed reads
      if (epi_any(!mbar_wait_cluster(&xfull[b], (i >> 1) & 1, a.err))) { ok = false; break; }
      // 3. P(i) goes into pbuf[b], so PE(i - 2) must be done with it (it is: tcgen05 work
      //    completes in issue order and L(i), issued after it, has completed)
      if (epi_any(i >= 2 && !mbar_wait(&pe_done[b], ((i - 2) >> 1) & 1, a.err))) { ok = false; break; }
      // 4. per-token statistics over the tile, P written as it is formed: warp tw, tokens
      //    8 tw + j, lane: vocab 4 lane .. +3
      const float* tb_ = theirs + b * kLmT * 128;
      uint8_t* pt = pbuf + b * kLmPBytes;
      int need = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int t = tw * 8 + j;
        const float4 x0 = *reinterpret_cast<const float4*>(mb + t * 128 + lane * 4);
        const float4 x1 = *reinterpret_cast<const float4*>(tb_ + t * 128 + lane * 4);
        float l[4] = {x0.x + x1.x, x0.y + x1.y, x0.z + x1.z, x0.w + x1.w};
        float mx = -INFINITY;
        int ax = 0x7fffffff;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = tile * 128 + lane * 4 + u;
          if (v >= a.V || v == a.mask_id) l[u] = -INFINITY;
          if (l[u] > mx) { mx = l[u]; ax = v; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float m2 = __shfl_xor_sync(0xffffffffu, mx, o);
          const int a2 = __shfl_xor_sync(0xffffffffu, ax, o);
          if (m2 > mx || (m2 == mx && a2 < ax)) { mx = m2; ax = a2; }
        }
        if (mx > mbest[j]) { mbest[j] = mx; arg[j] = ax; }
        float f = 1.f;
        if (i == 0) {
          ref[j] = mx;
        } else if (mx > ref[j] + kLmRescale) {
          f = expf(ref[j] - mx);
          ref[j] = mx;
          Z[j] *= f;
          A[j] *= f;
          need = 1;
        }
        if (lane == 0) fac[t] = f;
        float zs = 0.f, as = 0.f;
        __align__(8) __nv_bfloat16 hi[4], lo[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float p = (l[u] == -INFINITY) ? 0.f : expf(l[u] - ref[j]);
          zs += p;
          as += (p > 0.f) ? p * l[u] : 0.f;
          const float pw = (t < a.T) ? p : 0.f;
          hi[u] = f2bf(pw);
          lo[u] = f2bf(pw - bf2f(hi[u]));
        }
        if (!a.given) {
          *reinterpret_cast<uint2*>(pt + p_offset(t, lane * 4)) = *reinterpret_cast<const uint2*>(hi);
          *reinterpret_cast<uint2*>(pt + p_offset(32 + t, lane * 4)) = *reinterpret_cast<const uint2*>(lo);
        }
        Z[j] += warp_sum(zs);
        A[j] += warp_sum(as);
      }
      // 5. a raised reference rescales s (final up to tile i - 1: PE(i - 1) done) before
      //    PE(i) adds to it.  With a given P nothing is written or rescaled, but PE(i) still
      //    waits for this point, which keeps the MMA warp at most one PE ahead of these waits.
      const bool rescale = !a.given && epi_any(need != 0);  // also publishes fac[]
      if (rescale) {
        if (epi_any(i >= 1 && !mbar_wait(&pe_done[(i - 1) & 1], ((i - 1) >> 1) & 1, a.err))) { ok = false; break; }
        tc_fence_after();
        float fv[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) fv[t] = fac[t];
        for (int ch = 0; ch < CH; ++ch) {
          float sv[32];
          const uint32_t sa = tmem + ((uint32_t)(q * 32) << 16) + kLmSCol + ch * kLmT;
          tmem_ld32(sa, sv);
#pragma unroll
          for (int t = 0; t < 32; ++t) sv[t] *= fv[t];
          tmem_st32_f(sa, sv);
        }
        tc_fence_before();
      }
      fence_proxy_async_smem();  // generic-proxy writes of P visible to the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[b]);
    }
    // 6. outputs of the cluster: s half (every CTA), statistics (rank 0)
    if (ok && nt > 0) {
      const int last = nt - 1;
      if (et == 0) *flag = mbar_wait(&pe_done[last & 1], (last >> 1) & 1, a.err) ? 1 : 0;
      epi_bar();
      ok = *flag != 0;
      epi_bar();
      if (ok) {
        tc_fence_after();
        for (int ch = 0; ch < CH; ++ch) {
          float sv[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + kLmSCol + ch * kLmT, sv);
          float4* dst = reinterpret_cast<float4*>(a.part_s + ((size_t)clu * a.d + d0 + ch * 128 + row) * 32);
#pragma unroll
          for (int u = 0; u < 8; ++u) dst[u] = make_float4(sv[4 * u], sv[4 * u + 1], sv[4 * u + 2], sv[4 * u + 3]);
        }
        if (rank == 0 && lane == 0) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int t = tw * 8 + j;
            float* ps = a.part_stats + ((size_t)clu * 32 + t) * 4;
            ps[0] = ref[j];
            ps[1] = Z[j];
            ps[2] = A[j];
            ps[3] = mbest[j];
            a.part_arg[(size_t)clu * 32 + t] = arg[j];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer no longer writes into this CTA's shared memory
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Merge of the clusters: for token t, M = max_c r_c, Z = sum_c Z_c e^(r_c - M), lse = M + ln Z,
// maxprob = e^(max - lse), entropy = lse - A / Z, argmax from the lowest-index cluster holding
// the max; s[t][f] = sum_c e^(r_c - M) s_c[f][t] / Z (given P: plain sum).
// grid: d / 16 CTAs of 512 threads.  The per-token values are reduced in two steps (16 cluster
// chunks, then the chunks in order); then each warp takes one feature f (lane = token) and sums
// its clusters the same way (128 contiguous bytes per cluster).
constexpr int kLmfWarps = 16;
constexpr int kLmfSmem = (kLmMaxClusters * 32 + 4 * kLmfWarps * 32) * 4;
__global__ void __launch_bounds__(kLmfWarps * 32) k_lmf_combine(LmfArgs a, dlm_row_stats stats, float* s) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) float sm_f[];
  float(*w)[32] = reinterpret_cast<float(*)[32]>(sm_f);  // [clusters][32]
  float* cm = sm_f + kLmMaxClusters * 32;                 // [4][warps][32]
  __shared__ float Mt[32], iZ[32];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // 1. per token: thread (chunk = warp, token = lane) takes clusters chunk, chunk + 16, ...
  {
    const int t = lane, ch = warp;
    float4 ps[5];
    int nc = 0;
    float rmax = -INFINITY;
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      const int c = ch + k * kLmfWarps;
      if (c < a.n_clu) {
        ps[k] = *reinterpret_cast<const float4*>(a.part_stats + ((size_t)c * 32 + t) * 4);
        rmax = fmaxf(rmax, ps[k].x);
        nc = k + 1;
      }
    }
    cm[(0 * kLmfWarps + ch) * 32 + t] = rmax;
    __syncthreads();
    if (tid < 32) {
      float M = -INFINITY;
      for (int q = 0; q < kLmfWarps; ++q) M = fmaxf(M, cm[q * 32 + tid]);
      Mt[tid] = M;
    }
    __syncthreads();
    const float M = Mt[t];
    float zs = 0.f, as = 0.f, mx = -INFINITY, mc = 0.f;  // mc: cluster index of mx (as float)
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      if (k < nc) {
        const int c = ch + k * kLmfWarps;
        const float e = expf(ps[k].x - M);
        w[c][t] = a.given ? 1.f : e;
        zs += ps[k].y * e;
        as += ps[k].z * e;
        if (ps[k].w > mx) { mx = ps[k].w; mc = (float)c; }
      }
    }
    cm[(0 * kLmfWarps + ch) * 32 + t] = zs;
    cm[(1 * kLmfWarps + ch) * 32 + t] = as;
    cm[(2 * kLmfWarps + ch) * 32 + t] = mx;
    cm[(3 * kLmfWarps + ch) * 32 + t] = mc;
    __syncthreads();
    if (tid < 32) {
      float Z = 0.f, A = 0.f, bm = -INFINITY, bc = 1e30f;
      for (int q = 0; q < kLmfWarps; ++q) {  // chunks in order; ties -> lowest cluster index
        Z += cm[(0 * kLmfWarps + q) * 32 + tid];
        A += cm[(1 * kLmfWarps + q) * 32 + tid];
        const float m2 = cm[(2 * kLmfWarps + q) * 32 + tid], c2 = cm[(3 * kLmfWarps + q) * 32 + tid];
        if (m2 > bm || (m2 == bm && c2 < bc)) { bm = m2; bc = c2; }
      }
      iZ[tid] = (a.given ? 1.f : 1.f / Z) * a.s_scale;
      if (blockIdx.x == 0 && tid < a.T) {
        const float lse = Mt[tid] + logf(Z);
        stats.m[tid] = bm;
        stats.lse[tid] = lse;
        stats.maxprob[tid] = expf(bm - lse);
        stats.entropy[tid] = lse - A / Z;
        stats.argmax[tid] = a.part_arg[(size_t)(bc < (float)a.n_clu ? (int)bc : 0) * 32 + tid];  // NaN rows: cluster 0
      }
    }
  }
  __syncthreads();
  // 2. s[t][f] = iZ[t] sum_c w[c][t] s_c[f][t] for f = this CTA's 16 features, one per warp
  //    (lane = token); the clusters are summed in 16 interleaved chunks (c = q, q + 16, ...)
  //    whose sums are then added in chunk order, two chunks' loads in flight at a time
  const int f = blockIdx.x * kLmfWarps + warp;
  if (f >= a.d) return;
  const float* src = a.part_s + (size_t)f * 32 + lane;
  const size_t cs = (size_t)a.d * 32;  // one cluster's s block
  constexpr int kPer = (kLmMaxClusters + kLmfWarps - 1) / kLmfWarps;  // clusters per chunk
  float v = 0.f;
  for (int q = 0; q < kLmfWarps; q += 2) {
    float x[2][kPer];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int c = q + h + k * kLmfWarps;
        x[h][k] = c < a.n_clu ? __ldcg(src + (size_t)c * cs) : 0.f;
      }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int c = q + h + k * kLmfWarps;
        if (c < a.n_clu) acc = fmaf(w[c][lane], x[h][k], acc);
      }
      v += acc;
    }
  }
  if (lane < a.T) s[(size_t)lane * a.d + f] = v * iZ[lane];
}

// ------------------------------------------------------------------------------------------
// NVFP4 E: the same pass with E stored as e2m1 codes, e4m3 scales per 16 and an fp32 tensor
// scale S_E, and x quantized the same way per row (scale S_x[t]) by the last RMSNorm:
//   L  partial logits on the block-scaled FP4 tensor cores (kind::mxf4nvf4, 256 reduction
//      elements per stage: E codes 16 KB, x codes 4 KB, both operands' scales re-tiled for
//      tcgen05.cp), times S_E S_x[t] in the epilogue;
//   X  exchange and row statistics as above; P is written as f16 (one operand, N = 32);
//   PE s^T += E^T P with kind::f16 MMAs: four dequantisation warps re-read the E tile's codes
//      and scales (64 vocabulary rows x 128 features per step, from L2), turn them into f16
//      (e2m1 x e4m3 values are exact in f16) in the MN-major layout the MMA reads, and hand
//      them over through a two-slot ring.  The combine multiplies s by S_E.
// Warps: 0 lane 0 = producer of the L ring, lane 1 = producer of the PE code ring; 1 = MMA;
// 2..5 = statistics; 6..9 = dequantisation.
constexpr int kF4LmStages = 4;
constexpr int kF4LmStageBytes = 24576;  // E codes 16 KB | x codes 4 KB | E scales 2 KB | x scales 2 KB
constexpr int kF4LmPcStages = 4;
constexpr int kF4LmPcBytes = 5120;      // E codes [64 vocab][64 B] | E scales [64 vocab][16 B]
constexpr int kF4LmPhBytes = 16384;     // f16 E^T tile: 2 boxes [64 vocab][64 features]
constexpr int kF4LmPBytes = 8192;       // P f16 [32 tokens][128 vocab]: 2 atoms of 64
constexpr int kF4LmMaxChunks = 10;      // d / 2 <= 1280 (TMEM: 64 + 10 x 32 + 128 columns)
constexpr int kF4LmSCol = 64;           // TMEM column of the first s accumulator
constexpr int kF4LmSfCol = 384;         // TMEM columns of the scale-factor slots
constexpr int kF4LmThreads = 320;
constexpr float kF4PScale = 16.f;       // P is stored as f16 times this (p <= e^8 stays finite)
constexpr int kF4LmSmem = kF4LmStages * kF4LmStageBytes + kF4LmPcStages * kF4LmPcBytes + 2 * kF4LmPhBytes +
                          2 * kF4LmPBytes + 3 * kLmXBytes + 1024 + 1024;
static_assert(kF4LmSmem <= 232448, "fused NVFP4 LM head shared memory");

__device__ __forceinline__ uint32_t f16x2_from_e2m1x2(uint32_t two) {
  uint32_t h;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h) : "r"(two));
  return h;
}
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint32_t two) {
  uint32_t h;
  asm("{\n\t.reg .b16 b;\n\tcvt.u16.u32 b, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, b;\n\t}" : "=r"(h) : "r"(two));
  return h;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// Offset of element (row, v) of the f16 P tile (K-major B operand, 128-byte swizzle, two
// 64-wide atoms of 32 rows each).
__device__ __forceinline__ uint32_t p16_offset(int row, int v) {
  const int atom = v >> 6, c = v & 63;
  return (uint32_t)(atom * 4096 + row * 128 + ((((c >> 3) ^ (row & 7)) << 4) | ((c & 7) << 1)));
}

__global__ void __launch_bounds__(kF4LmThreads, 1)
k_lmhead_fused_f4(const __grid_constant__ CUtensorMap tec, const __grid_constant__ CUtensorMap tep,
                  const __grid_constant__ CUtensorMap tes, const __grid_constant__ CUtensorMap txc,
                  const uint8_t* __restrict__ sfe, const uint8_t* __restrict__ sfx, LmfArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;                                                  // L ring
  uint8_t* pcr = ring + kF4LmStages * kF4LmStageBytes;                   // PE code ring
  uint8_t* phr = pcr + kF4LmPcStages * kF4LmPcBytes;                     // f16 E^T ring [2]
  uint8_t* pbuf = phr + 2 * kF4LmPhBytes;                                // P [2]
  float* mine = (float*)(pbuf + 2 * kF4LmPBytes);                        // [128][32]
  float* theirs = mine + kLmT * 128;                                     // [2][128][32]
  uint64_t* bars = (uint64_t*)(theirs + 2 * kLmT * 128);
  uint64_t* full = bars;                          // [S]
  uint64_t* empty = full + kF4LmStages;           // [S]
  uint64_t* pc_full = empty + kF4LmStages;        // [PS]
  uint64_t* pc_empty = pc_full + kF4LmPcStages;   // [PS] (128 arrivals)
  uint64_t* ph_full = pc_empty + kF4LmPcStages;   // [2] (128 arrivals)
  uint64_t* ph_empty = ph_full + 2;               // [2] (MMA commit)
  uint64_t* accl_full = ph_empty + 2;             // [2]
  uint64_t* accl_empty = accl_full + 2;           // [2] (128 arrivals)
  uint64_t* p_ready = accl_empty + 2;             // [2] (4 arrivals)
  uint64_t* pe_done = p_ready + 2;                // [2]
  uint64_t* xfull = pe_done + 2;                  // [2] (128 remote arrivals)
  uint64_t* mma_done = xfull + 2;
  uint32_t* tmem_holder = (uint32_t*)(mma_done + 1);
  int* flag = (int*)(mma_done + 2);
  float* fac = (float*)(mma_done + 3);            // [32] rescale factors, then [4][32] quarter maxima

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const int clu = blockIdx.x / 2;
  const int dh = a.d / 2, d0 = (int)rank * dh;
  const int KB = dh / 256, CH = dh / 128, NB64 = a.d / 64;
  const int tb = lm_tile_begin(clu, a.n_tiles, a.n_clu), te = lm_tile_begin(clu + 1, a.n_tiles, a.n_clu);
  const int nt = te - tb;

  if (warp == 1 && lane == 0) {
    for (int i = 0; i < kF4LmStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < kF4LmPcStages; ++i) { mbar_init(&pc_full[i], 1); mbar_init(&pc_empty[i], 128); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ph_full[i], 128);
      mbar_init(&ph_empty[i], 1);
      mbar_init(&accl_full[i], 1);
      mbar_init(&accl_empty[i], 128);
      mbar_init(&p_ready[i], 4);
      mbar_init(&pe_done[i], 1);
      mbar_init(&xfull[i], 128);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tec);
    prefetch_tmap(&tep);
    prefetch_tmap(&tes);
    prefetch_tmap(&txc);
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_trigger();
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ---------------- L producer: per tile, KB stages of 256 reduction elements
    const uint64_t keep = l2_policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i) {
      const int tile = tb + i;
      for (int kb = 0; kb < KB && ok; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, a.err)) { ok = false; break; }
        uint8_t* st = ring + stage * kF4LmStageBytes;
        const int kc = (d0 + kb * 256) / 2;         // code byte of the stage's first element
        const int b64 = (d0 + kb * 256) / 64;       // its 64-element block
        mbar_arrive_expect_tx(&full[stage], kF4LmStageBytes);
        tma_load_2d_hint(st, &tec, &full[stage], kc, tile * 128, keep);
        tma_load_2d(st + 16384, &txc, &full[stage], kc, a.x_hi_row);
        bulk_load(st + 20480, sfe + ((size_t)tile * NB64 + b64) * 512, 2048, &full[stage]);
        bulk_load(st + 22528, sfx + (size_t)b64 * 512, 2048, &full[stage]);
        if (++stage == kF4LmStages) { stage = 0; phase ^= 1; }
      }
    }
    for (int i = 0; i < kF4LmStages && ok; ++i) {  // no copy left in flight
      if (!mbar_wait(&empty[stage], phase ^ 1, a.err)) break;
      if (++stage == kF4LmStages) { stage = 0; phase ^= 1; }
    }
  } else if (warp == 0 && lane == 1) {
    // ---------------- PE producer: per tile, CH x 2 steps of E codes [64 vocab][128 features]
    // and their scales (a 16-byte box holding this step's 8 scale bytes)
    const uint64_t drop = l2_policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i) {
      const int tile = tb + i;
      for (int ch = 0; ch < CH && ok; ++ch)
        for (int vh = 0; vh < 2 && ok; ++vh) {
          if (!mbar_wait(&pc_empty[stage], phase ^ 1, a.err)) { ok = false; break; }
          uint8_t* st = pcr + stage * kF4LmPcBytes;
          const int f0 = d0 + ch * 128;
          mbar_arrive_expect_tx(&pc_full[stage], kF4LmPcBytes);
          tma_load_2d_hint(st, &tep, &pc_full[stage], f0 / 2, tile * 128 + vh * 64, drop);
          tma_load_2d_hint(st + 4096, &tes, &pc_full[stage], (f0 / 16) & ~15, tile * 128 + vh * 64, drop);
          if (++stage == kF4LmPcStages) { stage = 0; phase ^= 1; }
        }
    }
    for (int i = 0; i < kF4LmPcStages && ok; ++i) {
      if (!mbar_wait(&pc_empty[stage], phase ^ 1, a.err)) break;
      if (++stage == kF4LmPcStages) { stage = 0; phase ^= 1; }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc_l = idesc_nvf4(128, kLmT);
    const uint32_t idesc_pe = idesc_f16(128, kLmT, true, false);
    int stage = 0, fs = 0;
    uint32_t phase = 0, fphase = 0;
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, a.err)) != 0;
    };
    auto mma_l = [&](int i) {
      const int b = i & 1;
      if (!wait_all(&accl_empty[b], ((i >> 1) & 1) ^ 1)) { ok = false; return; }
      tc_fence_after();
      const uint32_t dl = tmem + b * kLmT;
      for (int kb = 0; kb < KB; ++kb) {
        if (!wait_all(&full[stage], phase)) { ok = false; return; }
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + stage * kF4LmStageBytes);
        const uint32_t sfa_col = tmem + kF4LmSfCol + stage * 32, sfb_col = sfa_col + 16;
        const uint64_t ad = sw128_desc(sa, 16, 1024), bd = sw128_desc(sa + 16384, 16, 1024);
        const uint64_t fa = sf_desc(sa + 20480), fb = sf_desc(sa + 22528);
        if (elect_one()) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tmem_cp_32x128(sfa_col + 4 * j, fa + 32 * j);
            tmem_cp_32x128(sfb_col + 4 * j, fb + 32 * j);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_nvf4(dl, ad + 2 * j, bd + 2 * j, idesc_l, sfa_col + 4 * j, sfb_col + 4 * j, (kb | j) ? 1u : 0u);
          mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kF4LmStages) { stage = 0; phase ^= 1; }
      }
      if (elect_one()) mma_commit(&accl_full[b]);
      __syncwarp();
    };
    auto mma_pe = [&](int i) {
      const int b = i & 1;
      if (!wait_all(&p_ready[b], (i >> 1) & 1)) { ok = false; return; }
      tc_fence_after();
      const uint64_t pd = sw128_desc(smem_u32(pbuf + b * kF4LmPBytes), 16, 1024);
      for (int ch = 0; ch < CH; ++ch) {
        const uint32_t ds = tmem + kF4LmSCol + ch * kLmT;
        for (int vh = 0; vh < 2; ++vh) {
          if (!wait_all(&ph_full[fs], fphase)) { ok = false; return; }
          tc_fence_after();
          const uint64_t ad0 = sw128_desc(smem_u32(phr + fs * kF4LmPhBytes), 8192, 1024);
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k)  // 16 vocabulary rows (2048 B of E^T, 32 B of P) per step
              mma_bf16(ds, ad0 + 128 * k, pd + (vh * 4096 + k * 32) / 16, idesc_pe,
                       (i == 0 && vh == 0 && k == 0) ? 0u : 1u);
            mma_commit(&ph_empty[fs]);
          }
          __syncwarp();
          if (++fs == 2) { fs = 0; fphase ^= 1; }
        }
      }
      if (elect_one()) mma_commit(&pe_done[b]);
      __syncwarp();
    };
    for (int i = 0; i < nt && ok; ++i) {
      mma_l(i);
      if (ok && i >= 1) mma_pe(i - 1);
    }
    if (ok && nt > 0) mma_pe(nt - 1);
    if (elect_one()) {
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, a.err);
    }
    __syncwarp();
  } else if (warp >= 6) {
    // ---------------- dequantisation: thread dt owns vocabulary row dt / 2 and features
    // [64 (dt % 2), + 64) of each step's 128
    const int dt = threadIdx.x - 192, v = dt / 2, hf = dt % 2;
    int stage = 0, fs = 0;
    uint32_t phase = 0, fphase = 0;
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i)
      for (int ch = 0; ch < CH && ok; ++ch)
        for (int vh = 0; vh < 2 && ok; ++vh) {
          const int sofs = ((d0 + ch * 128) / 16) & 15;  // this step's first scale in the 16-byte box
          if (!mbar_wait(&ph_empty[fs], fphase ^ 1, a.err)) { ok = false; break; }
          if (!mbar_wait(&pc_full[stage], phase, a.err)) { ok = false; break; }
          const uint8_t* st = pcr + stage * kF4LmPcBytes;
          const uint4 c0 = *reinterpret_cast<const uint4*>(st + v * 64 + hf * 32);
          const uint4 c1 = *reinterpret_cast<const uint4*>(st + v * 64 + hf * 32 + 16);
          const uint32_t sc4 = *reinterpret_cast<const uint32_t*>(st + 4096 + v * 16 + sofs + hf * 4);
          const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          const uint32_t tile_b = smem_u32(phr + fs * kF4LmPhBytes) + hf * 8192 + v * 128;
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {  // 16 features: two code words, one scale
            const uint32_t sb = (sc4 >> (8 * blk)) & 0xFFu;
            const uint32_t sig = f16x2_from_e4m3x2(sb | (sb << 8));
            uint32_t o[8];
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const uint32_t word = cw[2 * blk + w];
#pragma unroll
              for (int q = 0; q < 4; ++q) o[4 * w + q] = hmul2(f16x2_from_e2m1x2((word >> (8 * q)) & 0xFFu), sig);
            }
            const int c = 2 * blk;  // 16-byte chunk of the 128-byte row (8 features each)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(tile_b + (((c) ^ (v & 7)) << 4)),
                         "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]) : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(tile_b + (((c + 1) ^ (v & 7)) << 4)),
                         "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7]) : "memory");
          }
          fence_proxy_async_smem();  // generic-proxy writes visible to the tensor cores
          // the code slot goes back only now that its values have been used: released right
          // after the loads were issued, the next TMA into the slot sometimes landed first
          mbar_arrive(&pc_empty[stage]);
          mbar_arrive(&ph_full[fs]);
          if (++stage == kF4LmPcStages) { stage = 0; phase ^= 1; }
          if (++fs == 2) { fs = 0; fphase ^= 1; }
        }
  } else if (warp >= 2) {
    // ---------------- statistics.  Phase 1 (thread = vocabulary row q*32 + lane of the tile): the
    // CTA's partial logits of the 32 tokens go to `mine` and to the peer's `theirs`, both laid
    // out [vocab 128][token 32] with the 16-byte chunks of a row rotated by (row & 7) (no bank
    // conflicts either way).  Phase 2 (thread = token t = lane, warp = vocabulary quarter q):
    // the full logits of its 32 rows, their max and lowest argmax, all in registers; the four
    // quarters agree on the tile max through shared memory, so every warp applies the same
    // running reference r_t; per-quarter sums Z_q, A_q and (max, argmax) are merged once,
    // after the last tile.
    const int q = warp % 4, row = q * 32 + lane, t = lane;
    const bool live = t < a.T;
    const float sct = live ? a.se * a.sx[t] : 0.f;  // S_E S_x[t]
    float ref = -INFINITY, Z = 0.f, A = 0.f, mbest = -INFINITY;
    int arg = 0x7fffffff;
    float* qmax = fac + 32;  // [4][32] quarter maxima of the current tile
    const uint32_t theirs_peer = map_peer(smem_u32(theirs), peer);
    const uint32_t xfull_peer = map_peer(smem_u32(xfull), peer);
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i) {
      const int b = i & 1, tile = tb + i;
      if (threadIdx.x == 64) *flag = mbar_wait(&accl_full[b], (i >> 1) & 1, a.err) ? 1 : 0;
      epi_bar();
      ok = *flag != 0;
      epi_bar();
      if (!ok) break;
      tc_fence_after();
      {
        float lp[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * kLmT, lp);
        tc_fence_before();
        mbar_arrive(&accl_empty[b]);
        float4* mrow = reinterpret_cast<float4*>(mine + row * 32);
        const uint32_t tpeer = theirs_peer + (uint32_t)((b * kLmT * 128 + row * 32) * 4);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 v4 = make_float4(lp[4 * u], lp[4 * u + 1], lp[4 * u + 2], lp[4 * u + 3]);
          const int cu = u ^ (row & 7);
          mrow[cu] = v4;
          st_cluster_v4(tpeer + (uint32_t)(cu * 16), v4);
        }
      }
      mbar_arrive_remote(xfull_peer + b * 8);
      if (epi_any(!mbar_wait_cluster(&xfull[b], (i >> 1) & 1, a.err))) { ok = false; break; }
      // P(i) goes into pbuf[b]: PE(i - 2) must be done with it
      if (epi_any(i >= 2 && !mbar_wait(&pe_done[b], ((i - 2) >> 1) & 1, a.err))) { ok = false; break; }
      const float* tb_ = theirs + b * kLmT * 128;
      float l[32];
      float mx = -INFINITY;
      int ax = 0x7fffffff;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int v = q * 32 + k, vv = tile * 128 + v;
        const int o = v * 32 + ((((t >> 2) ^ (v & 7))) << 2) + (t & 3);
        float x = (mine[o] + tb_[o]) * sct;
        if (vv >= a.V || vv == a.mask_id || !live) x = -INFINITY;
        l[k] = x;
        if (x > mx) { mx = x; ax = vv; }
      }
      if (mx > mbest) { mbest = mx; arg = ax; }
      qmax[q * 32 + t] = mx;
      epi_bar();
      const float tmx = fmaxf(fmaxf(qmax[t], qmax[32 + t]), fmaxf(qmax[64 + t], qmax[96 + t]));
      float f = 1.f;
      int need = 0;
      if (i == 0) {
        ref = tmx;
      } else if (tmx > ref + kLmRescale) {
        f = expf(ref - tmx);
        ref = tmx;
        Z *= f;
        A *= f;
        need = 1;
      }
      if (q == 0) fac[t] = f;
      uint32_t hw[16];
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        const float p0 = (l[k] == -INFINITY) ? 0.f : expf(l[k] - ref);
        const float p1 = (l[k + 1] == -INFINITY) ? 0.f : expf(l[k + 1] - ref);
        Z += p0;
        Z += p1;
        A += (p0 > 0.f) ? p0 * l[k] : 0.f;
        A += (p1 > 0.f) ? p1 * l[k + 1] : 0.f;
        const __half2 h = __floats2half2_rn(p0 * kF4PScale, p1 * kF4PScale);
        hw[k / 2] = *reinterpret_cast<const uint32_t*>(&h);
      }
      {  // row t of P, vocabulary 32 q .. 32 q + 31: four 16-byte chunks of atom q / 2
        uint8_t* prow = pbuf + b * kF4LmPBytes + (q >> 1) * 4096 + t * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(prow + ((((q & 1) * 4 + j) ^ (t & 7)) << 4)) =
              make_uint4(hw[4 * j], hw[4 * j + 1], hw[4 * j + 2], hw[4 * j + 3]);
      }
      // a raised reference rescales s (final up to tile i - 1: PE(i - 1) done) before PE(i)
      // adds to it; the barrier also ends this tile's reads of mine, theirs[b] and qmax
      const bool rescale = epi_any(need != 0);
      if (rescale) {
        if (epi_any(i >= 1 && !mbar_wait(&pe_done[(i - 1) & 1], ((i - 1) >> 1) & 1, a.err))) { ok = false; break; }
        tc_fence_after();
        for (int ch = 0; ch < CH; ++ch) {
          float sv[32];
          const uint32_t sa = tmem + ((uint32_t)(q * 32) << 16) + kF4LmSCol + ch * kLmT;
          tmem_ld32(sa, sv);
#pragma unroll
          for (int u = 0; u < 32; ++u) sv[u] *= fac[u];
          tmem_st32_f(sa, sv);
        }
        tc_fence_before();
      }
      fence_proxy_async_smem();  // generic-proxy writes of P visible to the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[b]);
    }
    if (ok && nt > 0) {
      const int last = nt - 1;
      if (threadIdx.x == 64) *flag = mbar_wait(&pe_done[last & 1], (last >> 1) & 1, a.err) ? 1 : 0;
      epi_bar();
      ok = *flag != 0;
      epi_bar();
      if (ok) {
        tc_fence_after();
        for (int ch = 0; ch < CH; ++ch) {
          float sv[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + kF4LmSCol + ch * kLmT, sv);
          float4* dst = reinterpret_cast<float4*>(a.part_s + ((size_t)clu * a.d + d0 + ch * 128 + row) * 32);
#pragma unroll
          for (int u = 0; u < 8; ++u) dst[u] = make_float4(sv[4 * u], sv[4 * u + 1], sv[4 * u + 2], sv[4 * u + 3]);
        }
        // the quarters' statistics of token t, merged in quarter order (`mine` is free now)
        float* ms = mine;  // [Z, A, max, argmax][quarter 4][token 32]
        ms[(0 * 4 + q) * 32 + t] = Z;
        ms[(1 * 4 + q) * 32 + t] = A;
        ms[(2 * 4 + q) * 32 + t] = mbest;
        reinterpret_cast<int*>(ms)[(3 * 4 + q) * 32 + t] = arg;
        epi_bar();
        if (rank == 0 && q == 0) {
          float zs = 0.f, as = 0.f, mb = -INFINITY;
          int ab = 0x7fffffff;
          for (int w = 0; w < 4; ++w) {
            zs += ms[(0 * 4 + w) * 32 + t];
            as += ms[(1 * 4 + w) * 32 + t];
            const float m = ms[(2 * 4 + w) * 32 + t];
            const int am = reinterpret_cast<const int*>(ms)[(3 * 4 + w) * 32 + t];
            if (m > mb || (m == mb && am < ab)) { mb = m; ab = am; }
          }
          float* ps = a.part_stats + ((size_t)clu * 32 + t) * 4;
          ps[0] = ref;
          ps[1] = zs;
          ps[2] = as;
          ps[3] = mb;
          a.part_arg[(size_t)clu * 32 + t] = ab;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                    uint32_t box_outer, char* err, size_t errlen) {
  return encode_tmap_2d(map, base, inner, outer, inner * 2, box_inner, box_outer, err, errlen);
}

}  // namespace

size_t lmhead_fused_scratch_bytes(int V, int d) {
  const int n_tiles = (V + 127) / 128;
  const int n_clu = n_tiles < kLmMaxClusters ? n_tiles : kLmMaxClusters;
  return (size_t)n_clu * 32 * 4 * sizeof(float) + (size_t)n_clu * 32 * sizeof(int) +
         (size_t)n_clu * d * 32 * sizeof(float) + 1024;
}

bool lmhead_fused_supported(int T, int d) {
  return T >= 1 && T <= kLmT && d % 256 == 0 && d / 256 <= kLmMaxChunks;
}

// x2: split bf16 pair of x2_rows rows: the T high halves from row hi_row, the T low halves
// from row lo_row.
cudaError_t lmhead_fused_launch(const void* x2, int x2_rows, int hi_row, int lo_row, const void* E,
                                const void* p_given, int T, int V, int d, int mask_id, dlm_row_stats stats,
                                float* s, void* scratch, int* d_err, cudaStream_t st, char* err,
                                size_t errlen) {
  // the 32-row boxes may reach past the buffer (TMA fills those rows with zeros, and columns
  // past T are dropped); the T live rows of each half must lie inside it
  if (hi_row % 8 || lo_row % 8 || hi_row < 0 || lo_row < 0 || hi_row + T > x2_rows || lo_row + T > x2_rows) {
    snprintf(err, errlen, "lm head: x rows %d / %d (+%d) of %d", hi_row, lo_row, T, x2_rows);
    return cudaErrorInvalidValue;
  }
  {
    static PerDeviceOnce once;
    const int r = once_on_current_device(once, [] {
      cudaError_t e = cudaFuncSetAttribute(k_lmhead_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, kLmSmem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_lmf_combine, cudaFuncAttributeMaxDynamicSharedMemorySize, kLmfSmem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_lmf_combine, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
      return (int)e;
    });
    if (r != 0) return (cudaError_t)r;
  }
  LmfArgs a{};
  a.V = V;
  a.d = d;
  a.T = T;
  a.mask_id = mask_id;
  a.x_hi_row = hi_row;
  a.x_lo_row = lo_row;
  a.n_tiles = (V + 127) / 128;
  a.n_clu = a.n_tiles < kLmMaxClusters ? a.n_tiles : kLmMaxClusters;
  a.given = p_given != nullptr;
  a.s_scale = 1.f;
  uint8_t* sc = (uint8_t*)scratch;
  a.part_stats = (float*)sc;
  a.part_arg = (int*)(sc + (size_t)a.n_clu * 32 * 4 * sizeof(float));
  a.part_s = (float*)(sc + (((size_t)a.n_clu * 32 * 5 * 4 + 255) & ~(size_t)255));
  a.err = d_err;
  CUtensorMap tek, tem, tx, tp;
  if (!encode_bf16_2d(&tek, E, d, V, 64, 128, err, errlen) || !encode_bf16_2d(&tem, E, d, V, 64, 64, err, errlen) ||
      !encode_bf16_2d(&tx, x2, d, x2_rows, 64, 32, err, errlen))
    return cudaErrorInvalidValue;
  if (p_given) {
    if (!encode_bf16_2d(&tp, p_given, V, T, 64, 32, err, errlen)) return cudaErrorInvalidValue;
  } else {
    tp = tx;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.n_clu);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = kLmSmem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_lmhead_fused, tek, tem, tx, tp, a);
  if (e != cudaSuccess) return e;
  return launch_k(k_lmf_combine, dim3((d + kLmfWarps - 1) / kLmfWarps), dim3(kLmfWarps * 32), kLmfSmem, st, a, stats, s);
}

bool lmhead_fused_f4_supported(int T, int d) {
  return T >= 1 && T <= kLmT && d % 512 == 0 && d / 256 <= kF4LmMaxChunks;
}

// E: NVFP4 codes [V][d/2], scales [V][d/16], tensor scale; sfe_tiled: its scales re-tiled for
// the block-scaled MMA; x: codes [x_rows][d/2] (token t in row t), tiled scales and row scales
// sx[T] as the quantizer of the last RMSNorm leaves them.
cudaError_t lmhead_fused_f4_launch(const dlm_nvfp4_matrix& E, const uint8_t* sfe_tiled, const uint8_t* xcodes,
                                   int x_rows, int x_row0, const uint8_t* xscales, const float* sx, int T, int V,
                                   int d, int mask_id, dlm_row_stats stats, float* s, void* scratch, int* d_err,
                                   cudaStream_t st, char* err, size_t errlen) {
  if (!lmhead_fused_f4_supported(T, d) || !E.codes || !E.scales || !sfe_tiled || !xcodes || !xscales || !sx ||
      x_row0 < 0 || x_row0 % 32 || x_row0 + T > x_rows) {
    snprintf(err, errlen, "nvfp4 lm head: unsupported arguments T=%d d=%d x rows %d + %d of %d", T, d, x_row0, T,
             x_rows);
    return cudaErrorInvalidValue;
  }
  {
    static PerDeviceOnce once;
    const int r = once_on_current_device(once, [] {
      cudaError_t e = cudaFuncSetAttribute(k_lmhead_fused_f4, cudaFuncAttributeMaxDynamicSharedMemorySize, kF4LmSmem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_lmf_combine, cudaFuncAttributeMaxDynamicSharedMemorySize, kLmfSmem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_lmf_combine, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
      return (int)e;
    });
    if (r != 0) return (cudaError_t)r;
  }
  LmfArgs a{};
  a.V = V;
  a.d = d;
  a.T = T;
  a.mask_id = mask_id;
  a.n_tiles = (V + 127) / 128;
  a.n_clu = a.n_tiles < kLmMaxClusters ? a.n_tiles : kLmMaxClusters;
  a.given = 0;
  a.se = E.tensor_scale;
  a.sx = sx + x_row0;      // the T rows' scales
  a.x_hi_row = x_row0;     // first row of their codes
  xscales += tok_scale_index(x_row0, 0, d);  // their group's plane of token scales
  a.s_scale = E.tensor_scale / kF4PScale;
  uint8_t* sc = (uint8_t*)scratch;
  a.part_stats = (float*)sc;
  a.part_arg = (int*)(sc + (size_t)a.n_clu * 32 * 4 * sizeof(float));
  a.part_s = (float*)(sc + (((size_t)a.n_clu * 32 * 5 * 4 + 255) & ~(size_t)255));
  a.err = d_err;
  CUtensorMap tec, tep, tes, txc;
  bool ok = encode_u8_2d(&tec, E.codes, (uint64_t)d / 2, V, 128, 128, true, err, errlen);
  ok = ok && encode_u8_2d(&tep, E.codes, (uint64_t)d / 2, V, 64, 64, false, err, errlen);
  ok = ok && encode_u8_2d(&tes, E.scales, (uint64_t)d / 16, V, 16, 64, false, err, errlen);
  ok = ok && encode_u8_2d(&txc, xcodes, (uint64_t)d / 2, x_rows, 128, 32, true, err, errlen);
  if (!ok) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.n_clu);
  cfg.blockDim = dim3(kF4LmThreads);
  cfg.dynamicSmemBytes = kF4LmSmem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_lmhead_fused_f4, tec, tep, tes, txc, sfe_tiled, xscales, a);
  if (e != cudaSuccess) return e;
  return launch_k(k_lmf_combine, dim3((d + kLmfWarps - 1) / kLmfWarps), dim3(kLmfWarps * 32), kLmfSmem, st, a, stats, s);
}

}  // namespace dlm

// dlm_attention.cu -- block-diffusion attention of one layer.
//
// The T queries of a block (positions L .. L+T-1) attend to every key of the prefix KV
// cache [0, L) and bidirectionally to all T keys of the block itself [L, L+T) (the block
// K/V are written to the cache before this kernel runs).  With `causal` set the query at
// position p sees keys [0, p] instead (prompt prefill).  [model card "QwenDLM-4B-ORL",
// "The paper's evaluation pipeline": the SDARPrefixKV block decoder]
//
// GQA packing: the G = Hq / Hkv query heads that share a KV head are stacked with the
// block's tokens into one set of T*G query rows, so one K/V tile read from HBM serves
// all of them.  A CTA owns 64 query rows (4 warps x 16) of one KV head and one split of
// the key range; the key range is split across CTAs (flash-decoding) so that short
// blocks still spread the KV stream over the SMs, and a combine kernel merges the splits
// with their (max, sum) statistics.  S = Q K^T and O = P V run on the tensor cores
// (mma.sync m16n8k16 bf16, fp32 accumulate); softmax is online in fp32 (base-2 exponent).
// The bf16 K/V tiles are staged by TMA (cp.async.bulk.tensor, 64 keys x 64 features per box,
// 128-byte swizzle; 64-byte for head_dim 32) into a double buffer completed on mbarriers.
#include <cstdio>
#include <cstring>

#include "dlm_device.cuh"
#include "dlm_internal.h"

namespace dlm {

constexpr int kAttnRows = 64;   // query rows per CTA
constexpr int kAttnKeys = 64;   // keys per tile
constexpr int kMinKeysPerSplit = 128;

constexpr int kKvStages = 3;  // bf16 cache: K/V ring depth (TMA)

template <int HD, bool FP8 = false>
struct AttnSmem {
  static constexpr int kTileBytes = 64 * HD * 2;
  // bf16 cache: a ring of kKvStages (K, V) tile pairs (Q goes to registers from global memory).
  // FP8 cache: Q + one bf16 K, V tile + the raw e4m3 K, V tiles and their 64 + 64 row scales
  // double-buffered
  static constexpr int kRawBytes = 2 * 64 * HD + 2 * 64 * 4;
  // + 1024: the tiles start on a 1024-byte boundary (the TMA swizzle atom)
  static constexpr int kBytes = (FP8 ? kTileBytes + 2 * kTileBytes + 2 * kRawBytes : 2 * kKvStages * kTileBytes) + 1024;
};

// Two e4m3 codes (low byte first) -> their values as a bf16 pair, exactly (e4m3 values are
// f16 values, and at most 4 significant bits fit bf16).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t two) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(two));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// Byte offset of 16-byte chunk `ch` (8 features) of row `row` in a [64][HD] bf16 tile, laid out
// as the TMA writes a box with the 128-byte swizzle (HD >= 64: rows of 128 B, HD = 128 as two
// [64][64] halves one after the other) or the 64-byte swizzle (HD = 32: rows of 64 B).  The
// swizzle spreads the 8 rows of an ldmatrix read over all banks.
template <int HD>
__device__ __forceinline__ uint32_t chunk_off(int row, int ch) {
  if constexpr (HD >= 64) return (uint32_t)((ch >> 3) * 8192 + row * 128 + (((ch & 7) ^ (row & 7)) << 4));
  else return (uint32_t)(row * 64 + (((ch & 3) ^ ((row >> 1) & 3)) << 4));
}
template <int HD>
__device__ __forceinline__ uint32_t tile_addr(uint32_t base, int row, int col) {
  // col in elements, multiple of 8 for chunk-aligned accesses
  return base + chunk_off<HD>(row, col >> 3) + (col & 7) * 2;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Number of key splits used for nkeys keys (the same rule on host and device).
__host__ __device__ __forceinline__ int attn_splits(int nkeys, int max_splits) {
  int s = (nkeys + kMinKeysPerSplit - 1) / kMinKeysPerSplit;
  if (s > max_splits) s = max_splits;
  if (s < 1) s = 1;
  return s;
}

template <int HD, bool FP8>
__global__ void __launch_bounds__(128)
k_bd_attention(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, AttnArgs a) {
  pdl_trigger();
  // bf16 cache: the prefix length (set between passes, never by a kernel of the pass) and the
  // K/V rows of the prefix [0, L) (written by earlier passes) do not depend on the previous
  // kernel, so the first prefix tiles are requested before waiting for it (below)
  if constexpr (FP8) pdl_wait();
  extern __shared__ uint8_t sm_raw[];
  uint8_t* const sm = (uint8_t*)(((uintptr_t)sm_raw + 1023) & ~(uintptr_t)1023);  // swizzle atoms
  __shared__ uint64_t kv_full[kKvStages];  // bf16 cache: the TMA K + V tiles of stage s have landed
  const int G = a.Hq / a.Hkv;
  const int rows_total = a.T * G;
  const int g = blockIdx.y, qt = blockIdx.x, split = blockIdx.z;
  const int L = a.pos0_dev ? *a.pos0_dev + a.pos_off : a.pos0;
  const int nkeys = L + a.T;
  // query token t sees keys [0, L + min(T, (t / blk + 1) blk)): causal is blk = 1, one
  // bidirectional block blk = T, a pending block followed by a new one blk = B
  const int blk = a.causal ? 1 : ((a.blk > 0 && a.blk < a.T) ? a.blk : a.T);
  auto key_end = [&](int t) { const int e = (t / blk + 1) * blk; return L + (e < a.T ? e : a.T); };
  const int nsplit = attn_splits(nkeys, a.max_splits);
  if (split >= nsplit) return;
  int chunk = (nkeys + nsplit - 1) / nsplit;
  chunk = (chunk + kAttnKeys - 1) / kAttnKeys * kAttnKeys;
  const int k0 = split * chunk;
  int k1 = min(nkeys, k0 + chunk);
  const int row0 = qt * kAttnRows;
  {
    // the last valid row of this CTA sees the most keys
    const int rlast = min(rows_total, row0 + kAttnRows) - 1;
    k1 = min(k1, key_end(rlast / G));
  }

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane / 4, tig = lane % 4;
  const uint32_t sQ = smem_u32(sm);  // FP8: the Q tile
  constexpr int TB = AttnSmem<HD>::kTileBytes;
  // bf16: stage s holds K at 2 s TB and V at (2 s + 1) TB; FP8: one bf16 K and V tile (after
  // the Q tile) converted from raw[buf] each step
  uint32_t sK[kKvStages], sV[kKvStages];
#pragma unroll
  for (int st = 0; st < kKvStages; ++st) {
    sK[st] = FP8 ? sQ + TB : sQ + 2 * st * TB;
    sV[st] = FP8 ? sQ + 2 * TB : sQ + (2 * st + 1) * TB;
  }
  uint8_t* const raw0 = sm + 3 * TB;  // FP8: [buf][K codes 64 x HD | V codes | K scales 64 | V scales 64]
  constexpr int RB = AttnSmem<HD, true>::kRawBytes;
  constexpr int CH = HD / 8;  // 16-byte chunks per row

  const int ntiles = (k1 > k0) ? (k1 - k0 + kAttnKeys - 1) / kAttnKeys : 0;
  if constexpr (!FP8) {
    if (threadIdx.x == 0) {
      for (int st = 0; st < kKvStages; ++st) mbar_init(&kv_full[st], 1);
      fence_mbar_init();
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
    }
  }

  auto load_kv = [&](int buf, int kt0) {
    if constexpr (FP8) {
      // raw e4m3 rows (HD bytes per key) and the 64 K / V row scales of the tile
      const uint8_t* kb8 = reinterpret_cast<const uint8_t*>(a.kc) + (size_t)g * a.max_ctx * HD;
      const uint8_t* vb8 = reinterpret_cast<const uint8_t*>(a.vc) + (size_t)g * a.max_ctx * HD;
      const uint32_t rb = smem_u32(raw0 + buf * RB);
      constexpr int C8 = HD / 16;  // 16-byte chunks per key
      for (int i = threadIdx.x; i < kAttnKeys * C8; i += 128) {
        const int r = i / C8, ch = i % C8;
        const int key = kt0 + r;
        const bool v = key < k1;
        const size_t off = (size_t)(v ? key : 0) * HD + ch * 16;
        cp_async16(rb + r * HD + ch * 16, kb8 + off, v);
        cp_async16(rb + kAttnKeys * HD + r * HD + ch * 16, vb8 + off, v);
      }
      if (threadIdx.x < 32) {  // 16 chunks of 4 scales each for K, then for V
        const int which = threadIdx.x / 16, ch = threadIdx.x % 16;
        const float* sc = (which ? a.vs : a.ks) + (size_t)g * a.max_ctx + kt0 + ch * 4;
        const bool v = kt0 + ch * 4 + 3 < k1;
        if (v) {
          cp_async16(rb + 2 * kAttnKeys * HD + which * 256 + ch * 16, sc, true);
        } else {
          // the tile's last keys: element-wise (zero past k1), no 16-byte read past the row
          float* d = reinterpret_cast<float*>(raw0 + buf * RB + 2 * kAttnKeys * HD + which * 256) + ch * 4;
          for (int u = 0; u < 4; ++u) d[u] = (kt0 + ch * 4 + u < k1) ? sc[u] : 0.f;
        }
      }
      cp_commit();
    } else {
      // one thread: the 64-key K and V boxes (rows g max_ctx + kt0 ..; rows past the cache's
      // end read as zeros, rows past k1 are masked, and V's are zeroed before use)
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&kv_full[buf], 2 * TB);
        const int y = g * a.max_ctx + kt0;
#pragma unroll
        for (int hh = 0; hh < (HD > 64 ? 2 : 1); ++hh) {
          tma_load_2d(sm + (sK[buf] - sQ) + hh * 8192, &tk, &kv_full[buf], hh * 64, y);
          tma_load_2d(sm + (sV[buf] - sQ) + hh * 8192, &tv, &kv_full[buf], hh * 64, y);
        }
      }
    }
  };
  // FP8: raw[buf] -> the bf16 K and V tiles, exactly (16 codes -> two 16-byte chunks)
  auto convert = [&](int buf) {
    const uint8_t* rk = raw0 + buf * RB;
    constexpr int C8 = HD / 16;
    for (int i = threadIdx.x; i < 2 * kAttnKeys * C8; i += 128) {
      const int which = i / (kAttnKeys * C8), j = i % (kAttnKeys * C8);
      const int r = j / C8, ch = j % C8;
      const uint4 src = *reinterpret_cast<const uint4*>(rk + which * kAttnKeys * HD + r * HD + ch * 16);
      const uint32_t w[4] = {src.x, src.y, src.z, src.w};
      uint32_t o[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        o[2 * u] = e4m3x2_to_bf16x2((uint16_t)(w[u] & 0xFFFFu));
        o[2 * u + 1] = e4m3x2_to_bf16x2((uint16_t)(w[u] >> 16));
      }
      const uint32_t base = which ? sV[0] : sK[0];
      const int c0 = ch * 2;  // 8-element (16-byte) chunk index of the first 8 values
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + chunk_off<HD>(r, c0)),
                   "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]) : "memory");
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + chunk_off<HD>(r, c0 + 1)),
                   "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7]) : "memory");
    }
  };

  // bf16: thread 0 requests the first kKvStages tiles; those that lie wholly in the prefix go
  // out before waiting for the previous kernel (its mbarrier init precedes them in the thread)
  int issued = 0;
  if constexpr (!FP8) {
    if (threadIdx.x == 0)
      while (issued < kKvStages && issued < ntiles && k0 + (issued + 1) * kAttnKeys <= L) {
        load_kv(issued, k0 + issued * kAttnKeys);
        ++issued;
      }
    pdl_wait();
    if (threadIdx.x == 0)
      for (; issued < kKvStages && issued < ntiles; ++issued) load_kv(issued, k0 + issued * kAttnKeys);
  }

  // ---- Q: row r <-> (token t = r / G, head g*G + r % G); the A fragments of this warp's 16 rows
  uint32_t qf[HD / 16][4];
  if constexpr (FP8) {
    for (int i = threadIdx.x; i < kAttnRows * CH; i += 128) {
      int r = i / CH, ch = i % CH;
      int R = row0 + r;
      bool v = R < rows_total;
      int t = v ? R / G : 0, h = g * G + (v ? R % G : 0);
      const __nv_bfloat16* src = a.q + ((size_t)t * a.Hq + h) * HD + ch * 8;
      cp_async16(sQ + chunk_off<HD>(r, ch), src, v);
    }
    cp_commit();
    if (ntiles > 0) load_kv(0, k0);
    cp_wait<1>();
    if (ntiles == 0) cp_wait<0>();
    __syncthreads();
#pragma unroll
    for (int ks = 0; ks < HD / 16; ++ks) {
      int r = warp * 16 + (lane % 16);
      int col = ks * 16 + (lane / 16) * 8;
      ldsm_x4(tile_addr<HD>(sQ, r, col), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
    }
  } else {
    // straight from global memory (L2): register j of k-step ks holds row gid (+ 8 for odd j),
    // features ks 16 + 8 (j / 2) + 2 tig and the next one
    const uint32_t* qrow[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int R = row0 + warp * 16 + gid + 8 * hf;
      qrow[hf] = R < rows_total
                     ? reinterpret_cast<const uint32_t*>(a.q + ((size_t)(R / G) * a.Hq + g * G + R % G) * HD)
                     : nullptr;
    }
#pragma unroll
    for (int ks = 0; ks < HD / 16; ++ks)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t* qr = qrow[j & 1];
        qf[ks][j] = qr ? __ldcg(qr + (ks * 16 + (j >> 1) * 8 + 2 * tig) / 2) : 0u;
      }
    __syncthreads();  // the ring's mbarriers are initialised for every thread
  }

  // per-thread rows: gid and gid + 8 of the warp's 16
  const int rA = row0 + warp * 16 + gid, rB = rA + 8;
  const int lim_A = key_end(min(rA, rows_total - 1) / G) - 1;
  const int lim_B = key_end(min(rB, rows_total - 1) / G) - 1;
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);  // log2(e) / sqrt(hd)
  float m_A = -INFINITY, m_B = -INFINITY, l_A = 0.f, l_B = 0.f;
  float acc[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  // a thread that gave up waiting for a tile waits no more (every thread still takes every
  // barrier); thread 0, which issues the loads, then issues no more of them
  bool timed_out = false;
  int fail_it = -1;
  for (int it = 0; it < ntiles; ++it) {
    const int buf = FP8 ? (it & 1) : it % kKvStages;
    const int kt0 = k0 + it * kAttnKeys;
    const float* ksc = nullptr;
    const float* vsc = nullptr;
    if constexpr (FP8) {
      cp_wait<0>();     // raw[buf] (the one group in flight) has landed for this thread
      __syncthreads();  // ... for every thread; and tile it - 1 is done with the bf16 tiles
      if (it + 1 < ntiles) load_kv(buf ^ 1, kt0 + kAttnKeys);  // overlaps this tile's work
      convert(buf);
      __syncthreads();
      ksc = reinterpret_cast<const float*>(raw0 + buf * RB + 2 * kAttnKeys * HD);
      vsc = ksc + kAttnKeys;
    } else {
      // the first kKvStages tiles went out in the prologue; tile it + kKvStages - 1 goes to the
      // stage of tile it - 1, which the barrier at the end of the previous step released
      const int nxt = it + kKvStages - 1;
      if (it >= 1 && nxt < ntiles && !timed_out) load_kv(nxt % kKvStages, k0 + nxt * kAttnKeys);
      if (!timed_out && !mbar_wait(&kv_full[buf], (uint32_t)(it / kKvStages) & 1u, a.err)) {
        timed_out = true;
        fail_it = it;
      }
      if (kt0 + kAttnKeys > k1) {
        // the tile's rows past k1 hold other positions or heads (any bits): P is 0 there, so V
        // must be finite; zero those rows (generic writes after the TMA's, ordered by the wait)
        const int r0 = k1 - kt0;
        for (int i = threadIdx.x; i < (kAttnKeys - r0) * CH; i += 128) {
          const int r = r0 + i / CH, ch = i % CH;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(sV[buf] + chunk_off<HD>(r, ch)), "r"(0u)
                       : "memory");
        }
        fence_async_shared();  // before any later TMA write of this buffer
        __syncthreads();
      }
    }
    const int kb = FP8 ? 0 : buf;  // bf16 tile of this step

    // S = Q K^T for 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < HD / 16; ++ks) {
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        // matrices: [keys nb2*16 + 0..7, hd ks*16 + 0..7], [.., +8], [keys +8.., hd 0..7], [.., +8]
        int m = lane / 8;
        int key = nb2 * 16 + (m / 2) * 8 + (lane % 8);
        int col = ks * 16 + (m % 2) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tile_addr<HD>(sK[kb], key, col), b0, b1, b2, b3);
        mma16816(s[nb2 * 2], qf[ks], b0, b1);
        mma16816(s[nb2 * 2 + 1], qf[ks], b2, b3);
      }
    }
    // FP8: the K row scale of each key multiplies its scores
    if constexpr (FP8) {
#pragma unroll
      for (int nb = 0; nb < 8; ++nb)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float sk = ksc[nb * 8 + tig * 2 + j];
          s[nb][j] *= sk;
          s[nb][2 + j] *= sk;
        }
    }
    // mask, running max
    float mx_A = -INFINITY, mx_B = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        int key = kt0 + nb * 8 + tig * 2 + j;
        float vA = (key <= lim_A && key < k1) ? s[nb][j] * sl2 : -INFINITY;
        float vB = (key <= lim_B && key < k1) ? s[nb][2 + j] * sl2 : -INFINITY;
        s[nb][j] = vA;
        s[nb][2 + j] = vB;
        mx_A = fmaxf(mx_A, vA);
        mx_B = fmaxf(mx_B, vB);
      }
    }
    mx_A = fmaxf(mx_A, __shfl_xor_sync(0xffffffffu, mx_A, 1));
    mx_A = fmaxf(mx_A, __shfl_xor_sync(0xffffffffu, mx_A, 2));
    mx_B = fmaxf(mx_B, __shfl_xor_sync(0xffffffffu, mx_B, 1));
    mx_B = fmaxf(mx_B, __shfl_xor_sync(0xffffffffu, mx_B, 2));
    const float mn_A = fmaxf(m_A, mx_A), mn_B = fmaxf(m_B, mx_B);
    const float base_A = (mn_A == -INFINITY) ? 0.f : mn_A;
    const float base_B = (mn_B == -INFINITY) ? 0.f : mn_B;
    const float al_A = exp2f(m_A - base_A), al_B = exp2f(m_B - base_B);
    m_A = mn_A;
    m_B = mn_B;
    float rs_A = 0.f, rs_B = 0.f;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      s[nb][0] = exp2f(s[nb][0] - base_A);
      s[nb][1] = exp2f(s[nb][1] - base_A);
      s[nb][2] = exp2f(s[nb][2] - base_B);
      s[nb][3] = exp2f(s[nb][3] - base_B);
      rs_A += s[nb][0] + s[nb][1];
      rs_B += s[nb][2] + s[nb][3];
    }
    l_A = l_A * al_A + rs_A;
    l_B = l_B * al_B + rs_B;
    // FP8: the V row scale of each key multiplies its weight in O = P V (the sums above stay
    // the softmax normaliser)
    if constexpr (FP8) {
#pragma unroll
      for (int nb = 0; nb < 8; ++nb)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float sv = vsc[nb * 8 + tig * 2 + j];
          s[nb][j] *= sv;
          s[nb][2 + j] *= sv;
        }
    }
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      acc[i][0] *= al_A;
      acc[i][1] *= al_A;
      acc[i][2] *= al_B;
      acc[i][3] *= al_B;
    }
    // O += P V, with P carried as a bf16 pair (hi + lo) so the weights keep ~16 bits
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {  // 16 keys per k-step
      uint32_t pa[4], pl[4];
      const float* p4[4] = {&s[2 * ks][0], &s[2 * ks][2], &s[2 * ks + 1][0], &s[2 * ks + 1][2]};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const __nv_bfloat162 hi = __floats2bfloat162_rn(p4[r][0], p4[r][1]);
        const float2 hf = __bfloat1622float2(hi);
        pa[r] = *reinterpret_cast<const uint32_t*>(&hi);
        pl[r] = pack_bf16(p4[r][0] - hf.x, p4[r][1] - hf.y);
      }
#pragma unroll
      for (int nb2 = 0; nb2 < HD / 16; ++nb2) {
        // matrices: [keys ks*16+0..7, hd nb2*16+0..7], [keys +8, ..], [keys 0..7, hd +8], [keys +8, hd +8]
        int m = lane / 8;
        int key = ks * 16 + (m % 2) * 8 + (lane % 8);
        int col = nb2 * 16 + (m / 2) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(tile_addr<HD>(sV[kb], key, col), b0, b1, b2, b3);
        mma16816(acc[nb2 * 2], pa, b0, b1);
        mma16816(acc[nb2 * 2 + 1], pa, b2, b3);
        mma16816(acc[nb2 * 2], pl, b0, b1);
        mma16816(acc[nb2 * 2 + 1], pl, b2, b3);
      }
    }
    __syncthreads();  // buffer `buf` is refilled two iterations later
  }
  if constexpr (!FP8) {
    // after a timeout no TMA may still be writing this CTA's shared memory when it leaves:
    // thread 0 had issued tiles up to fail_it + kKvStages - 1 at most
    if (threadIdx.x == 0 && fail_it >= 0)
      for (int j = fail_it; j < ntiles && j < fail_it + kKvStages; ++j)
        mbar_wait(&kv_full[j % kKvStages], (uint32_t)(j / kKvStages) & 1u, a.err);
  }

  // row sums across the quad
  l_A += __shfl_xor_sync(0xffffffffu, l_A, 1);
  l_A += __shfl_xor_sync(0xffffffffu, l_A, 2);
  l_B += __shfl_xor_sync(0xffffffffu, l_B, 1);
  l_B += __shfl_xor_sync(0xffffffffu, l_B, 2);

  const int Rows = a.Hkv * rows_total;
  for (int half = 0; half < 2; ++half) {
    const int R = half ? rB : rA;
    if (R >= rows_total) continue;
    const float mrow = half ? m_B : m_A, lrow = half ? l_B : l_A;
    const int t = R / G, h = g * G + R % G;
    if (nsplit == 1) {
      const float inv = lrow > 0.f ? 1.f / lrow : 0.f;
      __nv_bfloat16* dst = a.o + ((size_t)t * a.Hq + h) * HD;
#pragma unroll
      for (int nb = 0; nb < HD / 8; ++nb) {
        int col = nb * 8 + tig * 2;
        store_split(dst + col, a.o_lo, acc[nb][half * 2] * inv);
        store_split(dst + col + 1, a.o_lo, acc[nb][half * 2 + 1] * inv);
      }
    } else {
      const size_t prow = (size_t)split * Rows + (size_t)g * rows_total + R;
      float* dst = a.part_o + prow * HD;
#pragma unroll
      for (int nb = 0; nb < HD / 8; ++nb) {
        int col = nb * 8 + tig * 2;
        *reinterpret_cast<float2*>(dst + col) = make_float2(acc[nb][half * 2], acc[nb][half * 2 + 1]);
      }
      if (tig == 0) {
        a.part_ml[prow * 2 + 0] = mrow;
        a.part_ml[prow * 2 + 1] = lrow;
      }
    }
  }
}

// Merges the key splits: o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.  One CTA (128
// threads) per row: the split weights are formed once (thread s loads split s's (m, l)),
// then thread e loads O_s[e] of every split at once and sums them in split order.
__global__ void __launch_bounds__(128) k_attn_combine(AttnArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float wsp[64], wl[64];
  __shared__ float red[4];
  __shared__ float den_s;
  const int G = a.Hq / a.Hkv;
  const int rows_total = a.T * G;
  const int Rows = a.Hkv * rows_total;
  const int L = a.pos0_dev ? *a.pos0_dev + a.pos_off : a.pos0;
  const int nsplit = attn_splits(L + a.T, a.max_splits);
  if (nsplit == 1) return;
  const int row = blockIdx.x;  // over Rows
  if (row >= Rows) return;
  const int g = row / rows_total, R = row % rows_total;
  const int t = R / G, h = g * G + R % G;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  float ms = -INFINITY, ls = 0.f;
  if (tid < nsplit) {
    ms = a.part_ml[((size_t)tid * Rows + row) * 2];
    ls = a.part_ml[((size_t)tid * Rows + row) * 2 + 1];
  }
  float mx = warp_max(ls > 0.f ? ms : -INFINITY);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float w = (tid < nsplit && ls > 0.f) ? exp2f(ms - M) : 0.f;
  if (tid < 64) {
    wsp[tid] = w;
    wl[tid] = ls;  // the split's (m, l) were loaded by this thread above
  }
  __syncthreads();
  if (tid == 0) {
    float den = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) den = fmaf(wsp[sp], wl[sp], den);  // split order
    den_s = den;
  }
  __syncthreads();
  const float den = den_s;
  for (int e = tid; e < a.hd; e += blockDim.x) {
    float num = 0.f;
    const float* po = a.part_o + (size_t)row * a.hd + e;
    const size_t sstride = (size_t)Rows * a.hd;
    int sp = 0;
    for (; sp + 8 <= nsplit; sp += 8) {  // eight independent loads in flight
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = __ldcg(po + (size_t)(sp + u) * sstride);
#pragma unroll
      for (int u = 0; u < 8; ++u) num += wsp[sp + u] * x[u];
    }
    for (; sp < nsplit; ++sp) num += wsp[sp] * __ldcg(po + (size_t)sp * sstride);
    store_split(a.o + ((size_t)t * a.Hq + h) * a.hd + e, a.o_lo, den > 0.f ? num / den : 0.f);
  }
}

int attention_max_splits(int T, int Hq, int Hkv, int max_ctx) {
  const int G = Hq / Hkv;
  const int qtiles = (T * G + kAttnRows - 1) / kAttnRows;
  int ctas = qtiles * Hkv;
  int s = (2 * kSMs) / ctas;  // two CTAs per SM in a single wave (each CTA is latency-bound)
  int by_len = (max_ctx + T + kMinKeysPerSplit - 1) / kMinKeysPerSplit;
  if (s > by_len) s = by_len;
  if (s < 1) s = 1;
  if (s > 64) s = 64;
  return s;
}

size_t attention_scratch_bytes(int T, int Hq, int hd, int max_splits) {
  size_t rows = (size_t)T * Hq;
  return (size_t)max_splits * rows * (hd + 2) * sizeof(float);
}

template <int HD, bool FP8>
static cudaError_t attn_attr() {
  cudaError_t e = cudaFuncSetAttribute(k_bd_attention<HD, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       AttnSmem<HD, FP8>::kBytes);
  // the largest shared-memory carve-out, as the GEMMs (see ops_init_attributes)
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_bd_attention<HD, FP8>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
  return e;
}

int attention_init_attributes() {
  static PerDeviceOnce once;
  return once_on_current_device(once, [] {
    cudaError_t e = attn_attr<32, false>();
    if (e == cudaSuccess) e = attn_attr<64, false>();
    if (e == cudaSuccess) e = attn_attr<128, false>();
    if (e == cudaSuccess) e = attn_attr<32, true>();
    if (e == cudaSuccess) e = attn_attr<64, true>();
    if (e == cudaSuccess) e = attn_attr<128, true>();
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_attn_combine, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    return (int)e;
  });
}

int attention_split_cap(int T, int max_ctx) {
  int by_len = (max_ctx + T + kMinKeysPerSplit - 1) / kMinKeysPerSplit;
  return by_len < 64 ? (by_len < 1 ? 1 : by_len) : 64;
}

template <int HD>
static cudaError_t launch_hd(const AttnArgs& a, cudaStream_t s) {
  const int G = a.Hq / a.Hkv;
  dim3 grid((a.T * G + kAttnRows - 1) / kAttnRows, a.Hkv, a.max_splits);
  // bf16 cache: K and V of the layer as [Hkv * max_ctx][HD] for the TMA (boxes of 64 keys x
  // min(HD, 64) features); the FP8 cache is staged by cp.async (the maps are not used)
  CUtensorMap tk, tv;
  memset(&tk, 0, sizeof(tk));
  memset(&tv, 0, sizeof(tv));
  if (!a.ks) {
    char msg[160];
    const uint64_t rows = (uint64_t)a.Hkv * a.max_ctx;
    const uint32_t bi = HD < 64 ? HD : 64;
    const int sw = HD < 64 ? 64 : 128;
    if (!encode_tmap_2d_swizzle(&tk, a.kc, HD, rows, HD * 2, bi, kAttnKeys, sw, msg, sizeof(msg)) ||
        !encode_tmap_2d_swizzle(&tv, a.vc, HD, rows, HD * 2, bi, kAttnKeys, sw, msg, sizeof(msg)))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = a.ks ? launch_k(k_bd_attention<HD, true>, grid, dim3(128), AttnSmem<HD, true>::kBytes, s, tk, tv, a)
                       : launch_k(k_bd_attention<HD, false>, grid, dim3(128), AttnSmem<HD, false>::kBytes, s, tk, tv, a);
  if (e != cudaSuccess) return e;
  if (a.max_splits > 1) e = launch_k(k_attn_combine, dim3(a.Hkv * a.T * G), dim3(128), 0, s, a);
  return e;
}

cudaError_t attention_launch(const AttnArgs& a, cudaStream_t s) {
  switch (a.hd) {
    case 32: return launch_hd<32>(a, s);
    case 64: return launch_hd<64>(a, s);
    case 128: return launch_hd<128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dlm

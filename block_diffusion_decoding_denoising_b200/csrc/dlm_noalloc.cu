// dlm_noalloc.cu -- block-diffusion attention with library-owned scratch: an entry point
// for callers that cannot hand the library any device memory beyond the operands.
//
// dlm_bd_attention asks the caller for a scratch buffer (the split-KV partial results and
// a status word).  Some callers have no way to provide one: code that runs where device
// allocation is not allowed (a serving loop that has fixed its memory footprint up front,
// or a host thread without an allocator of its own) and that cannot keep a buffer
// between calls.  dlm_bd_attention_noalloc serves them: its scratch is a fixed array of
// kNoAllocScratchBytes in this file's static device memory, so a call allocates nothing.
//
// Limits and contract (also stated in include/dlm.h):
//  - calls whose split-KV partials do not fit in kNoAllocScratchBytes are rejected with
//    DLM_ENOMEM_WS before anything is launched;
//  - the first call on a device looks up the array's device address
//    (cudaGetSymbolAddress) and sets the kernels' shared-memory limits on that device;
//    make that first call before any stream capture is started on that device;
//  - the split partials need no initial value (every element read by the merge is written
//    first by the same call), so a call launches the attention kernels and nothing else;
//  - the array is shared by every call on a device: calls that may overlap in time (on
//    different streams, or from several host threads) race on it and must be serialised
//    by the caller.
#include <cuda_runtime.h>

#include <atomic>

#include "dlm_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device
constexpr size_t kNoAllocHeaderBytes = 256;                // unused head of the array (alignment)

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device (the name is only a host-side handle in
// host code), looked up by the first call on each device together with the kernels'
// attributes on that device.
std::atomic<void*> g_noalloc_ptr[dlm::kMaxDevices];
dlm::PerDeviceOnce g_noalloc_once;

cudaError_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int r = g_noalloc_once.run(dev, [dev] {
    void* p = nullptr;
    cudaError_t e2 = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e2 == cudaSuccess) e2 = (cudaError_t)dlm::attention_init_attributes();
    if (e2 == cudaSuccess) g_noalloc_ptr[dev].store(p, std::memory_order_release);
    return (int)e2;
  });
  if (r == dlm::PerDeviceOnce::kBadDevice) return cudaErrorInvalidDevice;
  if (r != 0) return (cudaError_t)r;
  *out = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  return *out ? cudaSuccess : cudaErrorInvalidDevice;
}

}  // namespace

extern "C" {

dlm_status dlm_bd_attention_noalloc(const void* d_q, const void* d_k_cache, const void* d_v_cache, void* d_o,
                                    int T, int L, int Hq, int Hkv, int hd, int max_ctx, int causal,
                                    void* stream) {
  if (!d_q || !d_k_cache || !d_v_cache || !d_o || T < 1 || L < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv ||
      !(hd == 32 || hd == 64 || hd == 128) || L + T > max_ctx)
    return DLM_EINVAL;
  const int splits = dlm::attention_max_splits(T, Hq, Hkv, max_ctx);
  if (dlm::attention_scratch_bytes(T, Hq, hd, splits) > kNoAllocScratchBytes - kNoAllocHeaderBytes)
    return DLM_ENOMEM_WS;
  void* base = nullptr;
  if (noalloc_scratch(&base) != cudaSuccess) return DLM_ECUDA;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned char* sc = (unsigned char*)base;
  dlm::AttnArgs a{};
  a.q = (const __nv_bfloat16*)d_q;
  a.kc = (const __nv_bfloat16*)d_k_cache;
  a.vc = (const __nv_bfloat16*)d_v_cache;
  a.o = (__nv_bfloat16*)d_o;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.hd = hd;
  a.max_ctx = max_ctx;
  a.pos0 = L;
  a.causal = causal ? 1 : 0;
  a.max_splits = splits;
  a.part_o = (float*)(sc + kNoAllocHeaderBytes);
  a.part_ml = a.part_o + (size_t)splits * T * Hq * hd;
  a.err = nullptr;
  if (dlm::attention_launch(a, s) != cudaSuccess) return DLM_ECUDA;
  return DLM_OK;
}

}  // extern "C"

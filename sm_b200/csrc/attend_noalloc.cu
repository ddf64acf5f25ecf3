// kvq_attend_noalloc: kvq_attend for callers that cannot hand the library a
// workspace because they cannot allocate device memory at call time -- for
// example code embedded in a serving engine that reserves all of its device
// memory when it starts and forbids allocation afterwards, or a hot loop
// where a cudaMalloc would synchronize the device and stall every stream.
//
// Its split-KV scratch is a fixed array compiled into this library instead of
// caller memory.  Each GPU that loads the library holds the array until the
// process exits.  The array is shared by every call on a device, so calls
// whose kernels may run at the same time on that device race on it; issue
// them on one stream, or order them.
#include <mutex>
#include <vector>

#include "kvq_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code
// the symbol names a host-side stand-in, not device memory, so its address
// must be asked for once per device with that device current.
kvq_status scratch_address(void** out) {
  static std::mutex mu;
  static std::vector<void*> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, nullptr);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
    cache[dev] = p;
  }
  *out = cache[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" {

kvq_status kvq_attend_noalloc(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                              const int32_t* lengths, int32_t H_q, int32_t Lq, float scale,
                              void* O, int32_t splits, void* stream) {
  // kvq_workspace_size returns 0 for invalid arguments; kvq_attend then
  // reports them.  Anything needing more than the fixed array is refused.
  const size_t need = kvq_workspace_size(cache, H_q, Lq, splits);
  if (need > KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  const kvq_status st = scratch_address(&scratch);
  if (st != KVQ_OK) return st;
  return kvq_attend(Q, q_dtype, cache, lengths, H_q, Lq, scale, O, scratch,
                    KVQ_NOALLOC_SCRATCH_BYTES, splits, stream);
}

size_t kvq_noalloc_scratch_bytes(void) { return KVQ_NOALLOC_SCRATCH_BYTES; }

}  // extern "C"

// C ABI entry points of libkvq.so: argument validation, dispatch, error word.
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "kvq_internal.cuh"

namespace kvq {

__device__ unsigned int g_error = 0;

unsigned int* error_word() {
  static std::mutex mu;
  static std::vector<unsigned int*> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, nullptr);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<unsigned int*>(p);
  }
  return cache[dev];
}

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

int sm_count() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

bool ensure_dynamic_smem(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<int, const void*>, size_t>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  for (auto& e : done)
    if (e.first.first == dev && e.first.second == kernel) {
      if (e.second >= bytes) return true;
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
          cudaSuccess)
        return false;
      e.second = bytes;
      return true;
    }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
      cudaSuccess)
    return false;
  done.push_back({{dev, kernel}, bytes});
  return true;
}

bool make_geometry(const kvq_cache* c, Geometry* g) {
  if (!c) return false;
  if (c->bits != 4 && c->bits != 8) return false;
  if (c->group < 2 || (c->group & 1)) return false;
  if (c->B < 1 || c->H_kv < 1 || c->N_cap < 1 || c->D < 1) return false;
  g->bits = c->bits;
  g->group = c->group;
  g->B = c->B;
  g->H_kv = c->H_kv;
  g->N_cap = c->N_cap;
  g->D = c->D;
  g->Np = (c->N_cap + c->group - 1) / c->group * c->group;
  g->Dp = (c->D + c->group - 1) / c->group * c->group;
  const size_t bytes_per_code_num = static_cast<size_t>(c->bits);
  g->k_codes_head = static_cast<size_t>(g->Np) * c->D * bytes_per_code_num / 8;
  g->k_scales_head = static_cast<size_t>(g->Np / c->group) * c->D;
  g->v_codes_head = static_cast<size_t>(c->N_cap) * g->Dp * bytes_per_code_num / 8;
  g->v_scales_head = static_cast<size_t>(c->N_cap) * (g->Dp / c->group);
  return true;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool fill_attend_args(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                             const int32_t* lengths, int32_t H_q, int32_t Lq, float scale,
                             void* O, void* ws, size_t ws_bytes, int32_t splits,
                             AttendArgs* a) {
  if (!make_geometry(cache, &a->g)) return false;
  if (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return false;
  if (H_q < 1 || Lq < 1 || H_q % cache->H_kv) return false;
  if (splits < 0) return false;
  a->Q = Q;
  a->q_dtype = q_dtype;
  a->k_codes = cache->k_codes;
  a->k_scales = cache->k_scales;
  a->v_codes = cache->v_codes;
  a->v_scales = cache->v_scales;
  a->lengths = lengths;
  a->H_q = H_q;
  a->Lq = Lq;
  a->scale = scale;
  a->O = O;
  a->workspace = ws;
  a->ws_bytes = ws_bytes;
  a->splits = splits;
  return true;
}

static const AttendImpl& choose(const AttendArgs& a) {
  if (const AttendImpl* c = chunk_attend_impl()) {
    if (c->applies(a)) return *c;
  }
  if (const AttendImpl* d = decode_attend_impl()) {
    if (d->applies(a)) return *d;
  }
  return generic_attend_impl();
}

}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_cache_sizes(int32_t bits, int32_t group, int32_t B, int32_t H_kv, int32_t N_cap,
                           int32_t D, size_t sizes[4]) {
  kvq_cache c{};
  c.bits = bits;
  c.group = group;
  c.B = B;
  c.H_kv = H_kv;
  c.N_cap = N_cap;
  c.D = D;
  Geometry g;
  if (!sizes || !make_geometry(&c, &g)) return KVQ_ERR_ARG;
  const size_t heads = static_cast<size_t>(B) * H_kv;
  sizes[0] = heads * g.k_codes_head;
  sizes[1] = heads * g.k_scales_head * sizeof(float);
  sizes[2] = heads * g.v_codes_head;
  sizes[3] = heads * g.v_scales_head * sizeof(float);
  return KVQ_OK;
}

size_t kvq_cache_bytes(const kvq_cache* cache) {
  if (!cache) return 0;
  size_t sizes[4];
  if (kvq_cache_sizes(cache->bits, cache->group, cache->B, cache->H_kv, cache->N_cap, cache->D, sizes) != KVQ_OK)
    return 0;
  return sizes[0] + sizes[1] + sizes[2] + sizes[3];
}

kvq_status kvq_pack(const void* K, const void* V, kvq_dtype in_dtype, int32_t t0, int32_t t1,
                    const kvq_cache* cache, void* stream) {
  PackArgs a{};
  if (!make_geometry(cache, &a.g)) return KVQ_ERR_ARG;
  if ((!K && !V) || !cache->k_codes || !cache->k_scales || !cache->v_codes || !cache->v_scales)
    return KVQ_ERR_ARG;
  if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16) return KVQ_ERR_ARG;
  if (t0 < 0 || t1 <= t0 || t1 > cache->N_cap) return KVQ_ERR_ARG;
  if (K && t0 % cache->group) return KVQ_ERR_ARG;
  const size_t esz = in_dtype == KVQ_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) % esz) return KVQ_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(cache->k_scales) | reinterpret_cast<uintptr_t>(cache->v_scales)) % 4)
    return KVQ_ERR_ALIGN;
  a.K = K;
  a.V = V;
  a.in_dtype = in_dtype;
  a.t0 = t0;
  a.t1 = t1;
  a.k_codes = cache->k_codes;
  a.k_scales = cache->k_scales;
  a.v_codes = cache->v_codes;
  a.v_scales = cache->v_scales;
  return launch_pack(a, static_cast<cudaStream_t>(stream));
}

size_t kvq_workspace_size(const kvq_cache* cache, int32_t H_q, int32_t Lq, int32_t splits) {
  AttendArgs a{};
  if (!fill_attend_args(nullptr, KVQ_BF16, cache, nullptr, H_q, Lq, 1.f, nullptr, nullptr, 0,
                        splits, &a))
    return 0;
  const AttendImpl& impl = choose(a);
  return impl.workspace(a);
}

// Every argument rule of the attend calls, checked on the host before any
// launch; on success *impl is the implementation that will run.
static kvq_status attend_prepare(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                                 const int32_t* lengths, int32_t H_q, int32_t Lq, float scale, void* O,
                                 void* workspace, size_t ws_bytes, int32_t splits, bool causal, AttendArgs* a,
                                 const AttendImpl** impl) {
  if (!fill_attend_args(Q, q_dtype, cache, lengths, H_q, Lq, scale, O, workspace, ws_bytes,
                        splits, a))
    return KVQ_ERR_ARG;
  a->causal = causal && Lq > 1;            // one query row at the last position sees every key
  if (!Q || !O || !lengths || !cache->k_codes || !cache->k_scales || !cache->v_codes ||
      !cache->v_scales)
    return KVQ_ERR_ARG;
  if (cache->D > 256) return KVQ_ERR_UNSUPPORTED;
  if (cache->B > 8192) return KVQ_ERR_UNSUPPORTED;
  if (!aligned16(cache->k_codes) || !aligned16(cache->k_scales) || !aligned16(cache->v_codes) ||
      !aligned16(cache->v_scales))
    return KVQ_ERR_ALIGN;
  // Q and O 16-byte aligned whatever their dtype, so that the kernel chosen
  // (and the workspace kvq_workspace_size reported) never depends on an address
  if (!aligned16(Q) || !aligned16(O)) return KVQ_ERR_ALIGN;
  if (reinterpret_cast<uintptr_t>(lengths) % 4) return KVQ_ERR_ALIGN;
  *impl = &choose(*a);
  const size_t need = (*impl)->workspace(*a);
  if (need > 0) {
    if (!workspace || ws_bytes < need) return KVQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KVQ_ERR_ALIGN;
  }
  return KVQ_OK;
}

static kvq_status attend_common(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                                const int32_t* lengths, int32_t H_q, int32_t Lq, float scale, void* O,
                                void* workspace, size_t ws_bytes, int32_t splits, bool causal, void* stream) {
  AttendArgs a{};
  const AttendImpl* impl = nullptr;
  const kvq_status st = attend_prepare(Q, q_dtype, cache, lengths, H_q, Lq, scale, O, workspace, ws_bytes,
                                       splits, causal, &a, &impl);
  if (st != KVQ_OK) return st;
  return impl->launch(a, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_attend(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                      const int32_t* lengths, int32_t H_q, int32_t Lq, float scale, void* O,
                      void* workspace, size_t ws_bytes, int32_t splits, void* stream) {
  return attend_common(Q, q_dtype, cache, lengths, H_q, Lq, scale, O, workspace, ws_bytes, splits, false,
                       stream);
}

kvq_status kvq_attend_causal(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                             const int32_t* lengths, int32_t H_q, int32_t Lq, float scale, void* O,
                             void* workspace, size_t ws_bytes, int32_t splits, void* stream) {
  return attend_common(Q, q_dtype, cache, lengths, H_q, Lq, scale, O, workspace, ws_bytes, splits, true,
                       stream);
}

kvq_status kvq_decode_step(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                           const int32_t* lengths, const void* K_tail, const void* V_new, kvq_dtype in_dtype,
                           int32_t H_q, float scale, void* O, void* workspace, size_t ws_bytes, int32_t splits,
                           void* stream) {
  AttendArgs a{};
  const AttendImpl* impl = nullptr;
  const kvq_status st = attend_prepare(Q, q_dtype, cache, lengths, H_q, 1, scale, O, workspace, ws_bytes,
                                       splits, false, &a, &impl);
  if (st != KVQ_OK) return st;
  if (!K_tail || !V_new || (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16)) return KVQ_ERR_ARG;
  const size_t esz = in_dtype == KVQ_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(K_tail) | reinterpret_cast<uintptr_t>(V_new)) % esz) return KVQ_ERR_ALIGN;
  AppendArgs ap{};
  ap.K_tail = K_tail;
  ap.V_new = V_new;
  ap.in_dtype = in_dtype;
  ap.lengths = lengths;
  ap.g = a.g;
  ap.k_codes = cache->k_codes;
  ap.k_scales = cache->k_scales;
  ap.v_codes = cache->v_codes;
  ap.v_scales = cache->v_scales;
  if (impl == decode_attend_impl()) {
    // the tuned decode kernel appends the new tokens itself: one launch less
    a.K_tail_step = K_tail;
    a.V_new_step = V_new;
    a.step_dtype = in_dtype;
    return impl->launch(a, static_cast<cudaStream_t>(stream));
  }
  if (append_smem_bytes(a.g) > 227 * 1024 || a.g.H_kv > 65535) return KVQ_ERR_UNSUPPORTED;
  const kvq_status ast = launch_append(ap, static_cast<cudaStream_t>(stream));
  if (ast != KVQ_OK) return ast;
  return impl->launch(a, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_selftest_timeout(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                                const int32_t* lengths, int32_t H_q, float scale, void* O, void* workspace,
                                size_t ws_bytes, int32_t splits, int32_t lose_block, uint32_t wait_ms,
                                void* stream) {
  AttendArgs a{};
  const AttendImpl* impl = nullptr;
  const kvq_status st = attend_prepare(Q, q_dtype, cache, lengths, H_q, 1, scale, O, workspace, ws_bytes,
                                       splits, false, &a, &impl);
  if (st != KVQ_OK) return st;
  if (impl != decode_attend_impl()) return KVQ_ERR_UNSUPPORTED;
  if (lose_block < 0 || wait_ms < 1 || wait_ms > 10000) return KVQ_ERR_ARG;
  a.test_lose_block = lose_block;
  a.test_wait_ns = static_cast<unsigned long long>(wait_ms) * 1000000ull;
  return impl->launch(a, static_cast<cudaStream_t>(stream));
}

static bool fill_window(const void* K_win, const void* V_win, kvq_dtype win_dtype,
                        const int32_t* win_lengths, int32_t W_cap, AttendArgs* a) {
  if (win_dtype != KVQ_F32 && win_dtype != KVQ_BF16) return false;
  if (W_cap < 1) return false;
  a->K_win = K_win;
  a->V_win = V_win;
  a->win_dtype = win_dtype;
  a->win_lengths = win_lengths;
  a->W_cap = W_cap;
  return true;
}

size_t kvq_workspace_size_window(const kvq_cache* cache, int32_t H_q, int32_t Lq, int32_t splits) {
  AttendArgs a{};
  if (!fill_attend_args(nullptr, KVQ_BF16, cache, nullptr, H_q, Lq, 1.f, nullptr, nullptr, 0,
                        splits, &a))
    return 0;
  static const int32_t dummy = 0;
  a.win_lengths = &dummy;                // only "has a window" matters for the size
  a.W_cap = 1;
  const AttendImpl& impl = choose(a);
  return impl.workspace(a);
}

kvq_status kvq_attend_window(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                             const int32_t* lengths, const void* K_win, const void* V_win,
                             kvq_dtype win_dtype, const int32_t* win_lengths, int32_t W_cap,
                             int32_t H_q, int32_t Lq, float scale, void* O, void* workspace,
                             size_t ws_bytes, int32_t splits, void* stream) {
  AttendArgs a{};
  if (!fill_attend_args(Q, q_dtype, cache, lengths, H_q, Lq, scale, O, workspace, ws_bytes,
                        splits, &a))
    return KVQ_ERR_ARG;
  if (!fill_window(K_win, V_win, win_dtype, win_lengths, W_cap, &a)) return KVQ_ERR_ARG;
  if (!Q || !O || !lengths || !K_win || !V_win || !win_lengths || !cache->k_codes || !cache->k_scales ||
      !cache->v_codes || !cache->v_scales)
    return KVQ_ERR_ARG;
  if (cache->D > 256) return KVQ_ERR_UNSUPPORTED;
  if (cache->B > 8192) return KVQ_ERR_UNSUPPORTED;
  if (!aligned16(cache->k_codes) || !aligned16(cache->k_scales) || !aligned16(cache->v_codes) ||
      !aligned16(cache->v_scales))
    return KVQ_ERR_ALIGN;
  if (!aligned16(Q) || !aligned16(O)) return KVQ_ERR_ALIGN;
  const size_t wsz = win_dtype == KVQ_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(K_win) | reinterpret_cast<uintptr_t>(V_win)) % wsz) return KVQ_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(lengths) | reinterpret_cast<uintptr_t>(win_lengths)) % 4) return KVQ_ERR_ALIGN;
  const AttendImpl& impl = choose(a);
  const size_t need = impl.workspace(a);
  if (!workspace || ws_bytes < need) return KVQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return KVQ_ERR_ALIGN;
  return impl.launch(a, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_check(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int h = 0;
  if (cudaMemcpyFromSymbolAsync(&h, g_error, sizeof(h), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return KVQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
  if (h != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return KVQ_ERR_CUDA;
  }
  return static_cast<kvq_status>(h);
}

const char* kvq_strerror(kvq_status status) {
  switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_ARG: return "invalid argument";
    case KVQ_ERR_LENGTH: return "sequence length outside its valid range (1..N_cap, or a window or causal rule)";
    case KVQ_ERR_ALIGN: return "pointer not suitably aligned";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    case KVQ_ERR_DEVICE: return "kernel reported an internal inconsistency";
    case KVQ_ERR_TIMEOUT: return "bounded wait inside a kernel ran out";
    case KVQ_ERR_UNSUPPORTED: return "arguments outside what this library implements";
  }
  return "unknown status";
}

uint64_t kvq_launch_count(void) { return g_launches.load(); }

const char* kvq_attend_kernel_name(const kvq_cache* cache, int32_t H_q, int32_t Lq) {
  AttendArgs a{};
  if (!fill_attend_args(nullptr, KVQ_BF16, cache, nullptr, H_q, Lq, 1.f, nullptr, nullptr, 0, 0,
                        &a))
    return "invalid";
  return choose(a).name;
}

}  // extern "C"

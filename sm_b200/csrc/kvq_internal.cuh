// Internal declarations shared by the CUDA sources of libkvq.so.
#pragma once
#include <utility>

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/kvq.h"

namespace kvq {

// ---------------------------------------------------------------------------
// device error word (one per device, per loaded library)
// ---------------------------------------------------------------------------
// Device address of the error word of the current device (host; cached per
// device).  Kernels receive it as a parameter and record the first error.
unsigned int* error_word();

__device__ __forceinline__ void record_error(unsigned int* err, kvq_status s) {
  atomicCAS(err, 0u, static_cast<unsigned int>(s));
}

// host launch counter
void count_launch(int n = 1);

// SM count of the current device (cached per device)
int sm_count();

// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes) on the
// current device unless an equal or larger value was already set there:
// the attribute call costs host time on every launch otherwise.
bool ensure_dynamic_smem(const void* kernel, size_t bytes);

// ---------------------------------------------------------------------------
// cache geometry
// ---------------------------------------------------------------------------
struct Geometry {
  int bits, group, B, H_kv, N_cap, D;
  int Np, Dp;                      // padded token / feature counts
  size_t k_codes_head, k_scales_head, v_codes_head, v_scales_head;  // per (b,h), in elements
};

bool make_geometry(const kvq_cache* c, Geometry* g);

// ---------------------------------------------------------------------------
// programmatic dependent launch
// ---------------------------------------------------------------------------
// Every kernel of the library is launched with launch_pdl, so its CTAs may
// become resident while the previous kernel on the stream drains, and starts
// with griddep_wait() -- which returns once every earlier grid on the stream
// has completed and its memory is visible -- before any global-memory
// access; it then lets the next kernel be scheduled.  Without a predecessor
// (or without the launch attribute) both are no-ops.  Two kernels always run
// right after one of the library's own, which has waited for every grid
// before it by the time it lets them be scheduled, and read some of the
// call's inputs (which no kernel of the library writes) before their own
// wait, through the L2 (ld.global.cg): the split merge computes its plan
// from the lengths, and the window kernel (griddep_release / griddep_join
// below) does all its work.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The split form, for a kernel launched right after one that started with
// griddep_wait() (so every grid before that one has completed by the time this
// one is scheduled), which reads only the call's inputs and writes workspace
// that no grid in flight touches: it lets the next kernel be scheduled at once
// (griddep_release), runs beside its predecessor, and waits for it only at
// its end (griddep_join), so that its own completion still implies the
// predecessor's -- the kernel after it reads what both wrote.
__device__ __forceinline__ void griddep_release() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_join() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// dtype helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float load_as_f32(const void* p, size_t i, int dtype) {
  if (dtype == KVQ_F32) return static_cast<const float*>(p)[i];
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

__device__ __forceinline__ void store_from_f32(void* p, size_t i, float v, int dtype) {
  if (dtype == KVQ_F32) static_cast<float*>(p)[i] = v;
  else static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

// ---------------------------------------------------------------------------
// work plan over the concatenated (b, h, block) list
//
// Blocks of BT tokens, ordered b-major, then h, then block index.  CTA c of
// `ctas` takes the contiguous global blocks [c*P, min((c+1)*P, T)), with
// P = ceil(T / ctas).  Whenever the CTA leaves a (b, h) it has not covered
// whole, it writes a partial (m, z, u) into slot (c + bh): along the monotone
// walk of (c, bh) pairs that sum is strictly increasing, so slots are unique
// and fewer than ctas + B*H_kv.
// ---------------------------------------------------------------------------
struct PlanArgs {
  const int32_t* lengths;
  int B, H_kv, N_cap, BT, ctas;
};

// per-sequence block count with the length clamped to [0, N_cap]
__device__ __forceinline__ int seq_blocks(int len, int n_cap, int bt) {
  len = len < 0 ? 0 : (len > n_cap ? n_cap : len);
  return (len + bt - 1) / bt;
}

// Merge partial states of a split (b, h) and write the output rows.
struct MergeArgs {
  const float* partials;           // row-major: [slots][R_pad][D + 2] : m, z, u[D]
                                   // feature-major: [slots][R_pad / 32][D + 2][32]
  const int32_t* lengths;
  void* O;
  int o_dtype;
  int B, H_kv, N_cap, BT, ctas;
  int R, R_pad, D;                 // rows per (b,h) and the padded row count of a slot
  int G, Lq;                       // query heads per KV head, rows per query head
  bool feature_major;              // partial layout (rows contiguous per field)
  bool causal;                     // causal rows: a length below Lq leaves rows without keys
  int extra_slots;                 // per-head plan slots past the last block (the decode step's
                                   // append, warp_block_prefix's extra); 0 elsewhere
  // recent-token window (kvq_attend_window); win_lengths == nullptr: none.
  // With a window every (b, h) is merged: its window state sits in slot
  // win_slot0 + b * H_kv + h, and no worker wrote an output row itself.
  const int32_t* win_lengths;
  int W_cap;
  long long win_slot0;
};
kvq_status launch_merge(const MergeArgs& a, cudaStream_t s);

// The window's partial state (m, z, u) of every row of every (b, h), written
// into slot slot0 + b * H_kv + h of the caller's partial layout: element
// (row r, field f) of a slot at (r / 32) * row_chunk_stride + (r % 32) *
// row_stride + f * field_stride (field 0 = m in natural-log units, 1 = z,
// 2 + d = u[d]).
struct WindowArgs {
  const void* Q;
  int q_dtype;
  const void* K_win;
  const void* V_win;
  int win_dtype;
  const int32_t* win_lengths;
  int W_cap;
  int B, H_kv, G, Lq, D;
  float scale;
  float* partials;
  long long slot0, slot_stride, row_stride, row_chunk_stride, field_stride;
};
kvq_status launch_window(const WindowArgs& w, cudaStream_t s);

struct AttendArgs;
// After an implementation's packed-cache kernel: when the call has a window,
// launch the window kernel into slots [slot0, slot0 + B * H_kv) of
// `partials` (laid out with the given strides, in floats) and point the
// merge at them.  Without a window it does nothing.
kvq_status add_window(const AttendArgs& a, float* partials, long long slot0, long long slot_stride,
                      long long row_stride, long long row_chunk_stride, long long field_stride, MergeArgs* m,
                      cudaStream_t s);

// ---------------------------------------------------------------------------
// kernels' host launchers
// ---------------------------------------------------------------------------
struct PackArgs {
  const void* K;
  const void* V;
  int in_dtype;
  int t0, t1;
  Geometry g;
  uint8_t* k_codes;
  float* k_scales;
  uint8_t* v_codes;
  float* v_scales;
};
kvq_status launch_pack(const PackArgs& a, cudaStream_t s);

// Decode-step append (kvq_decode_step): re-pack the K group holding each
// sequence's new token t = lengths[b] - 1 from its float rows, pack V row t.
struct AppendArgs {
  const void* K_tail;              // [B, H_kv, g, D]
  const void* V_new;               // [B, H_kv, D]
  int in_dtype;
  const int32_t* lengths;
  Geometry g;
  uint8_t* k_codes;
  float* k_scales;
  uint8_t* v_codes;
  float* v_scales;
};
size_t append_smem_bytes(const Geometry& g);
kvq_status launch_append(const AppendArgs& a, cudaStream_t s);

struct AttendArgs {
  const void* Q;
  int q_dtype;
  Geometry g;
  const uint8_t* k_codes;
  const float* k_scales;
  const uint8_t* v_codes;
  const float* v_scales;
  const int32_t* lengths;
  int H_q, Lq;
  float scale;
  void* O;
  void* workspace;
  size_t ws_bytes;
  int splits;
  bool causal;                     // kvq_attend_causal: query i of Lq reads keys [0, len - Lq + i]
  // recent-token window (kvq_attend_window); win_lengths == nullptr: none
  const void* K_win;
  const void* V_win;
  int win_dtype;
  const int32_t* win_lengths;
  int W_cap;
  // self-test of the tuned decode kernel's timeout path (kvq_selftest_timeout):
  // worker 0 loses the completion of its test_lose_block-th block and every
  // wait is bounded by test_wait_ns; -1 / 0: none, the default limit
  int test_lose_block = -1;
  unsigned long long test_wait_ns = 0;
  // kvq_decode_step: the new tokens' K group rows and V rows, appended by the
  // tuned decode kernel itself (nullptr: no append)
  const void* K_tail_step = nullptr;
  const void* V_new_step = nullptr;
  int step_dtype = 0;
};

// Workspace of an implementation whose packed partials fill `slots` slots of
// `slot_bytes`: a window adds one slot per (b, h) after them.
inline size_t with_window_slots(const AttendArgs& a, size_t slots, size_t slot_bytes) {
  const size_t win = a.win_lengths ? static_cast<size_t>(a.g.B) * static_cast<size_t>(a.g.H_kv) : 0;
  return (slots + win) * slot_bytes;
}

// One implementation of kvq_attend: how much workspace it needs and how to
// launch it.  `applies` says whether it handles these arguments.
struct AttendImpl {
  const char* name;
  bool (*applies)(const AttendArgs&);
  size_t (*workspace)(const AttendArgs&);
  kvq_status (*launch)(const AttendArgs&, cudaStream_t);
};

const AttendImpl& generic_attend_impl();
const AttendImpl* decode_attend_impl();     // tuned decode; nullptr if not built
const AttendImpl* chunk_attend_impl();      // tensor-core chunk; nullptr if not built

// Partial-slot bound shared by every split implementation.
inline size_t partial_slots(int ctas, int B, int H_kv) {
  return static_cast<size_t>(ctas) + static_cast<size_t>(B) * static_cast<size_t>(H_kv);
}

}  // namespace kvq

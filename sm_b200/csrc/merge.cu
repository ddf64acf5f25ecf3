// Split-KV merge: the (m, z, u) states several CTAs computed for one (b, h)
// combine with the same rescale rule as the block merge -- m = max of the
// parts, each part scaled by exp(m_part - m) before z and u are summed, a part
// without a valid key (z = 0) skipped -- then O = u / z ("Block KV decoding:
// less workspace, more time", huhohoo.com/en/docs/llm/kv-block-decode-cost,
// section "Do not average independently normalized blocks"; "给长前缀列一张有
// 单位的资源账本", section "FlashAttention为什么不必保存整张热图").
//
// Two layouts of the per-CTA partial states.  Row-major ([slot][row][m, z,
// u...]), for the few-row decode kernels: one CTA per (b, h), a warp per row.
// Feature-major ([slot][field][row]), for the many-row chunk kernel: one CTA
// per (b, h) and 32-row chunk, lane = row so every partial read is a
// coalesced 128-byte line, the merged tile staged in shared memory and
// written out as whole rows.
//
// A (b, h) that one CTA covered whole was already written by that CTA and is
// skipped here.  The merge also owns the sequences with no valid key: it
// records KVQ_ERR_LENGTH and writes zeros.
#include "kvq_internal.cuh"
#include "plan.cuh"

namespace kvq {
namespace {

struct MergeParams {
  MergeArgs a;
  unsigned int* err;
};

__global__ void __launch_bounds__(128) merge_kernel(MergeParams mp) {
  extern __shared__ int s_pre[];                 // [B + 1]
  const MergeArgs& a = mp.a;
  if (threadIdx.x < 32) warp_block_prefix(a.lengths, a.B, a.N_cap, a.BT, s_pre);
  __syncthreads();
  const int H = a.H_kv;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int D = a.D;
  const long long row_base = (static_cast<long long>(b) * H * a.G + static_cast<long long>(h) * a.G) * a.Lq;
  const int raw_len = a.lengths[b];
  if (h == 0 && threadIdx.x == 0 && (raw_len < 1 || raw_len > a.N_cap)) record_error(mp.err, KVQ_ERR_LENGTH);
  const int nb = s_pre[b + 1] - s_pre[b];
  if (nb == 0) {
    for (int idx = threadIdx.x; idx < a.R * D; idx += blockDim.x)
      store_from_f32(a.O, row_base * D + idx, 0.f, a.o_dtype);
    return;
  }
  const CtaRange cr = cta_range(s_pre, a.B, H, a.ctas, 0);
  const long long S = static_cast<long long>(H) * s_pre[b] + static_cast<long long>(h) * nb;
  const long long E = S + nb;
  const long long c_first = S / cr.P, c_last = (E - 1) / cr.P;
  if (c_first == c_last) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int W = D + 2;
  for (int r = warp; r < a.R; r += nwarps) {
    float m = -INFINITY;
    for (long long c = c_first; c <= c_last; ++c) {
      const float* part = a.partials + ((c + bh) * a.R_pad + r) * W;
      if (part[1] > 0.f) m = fmaxf(m, part[0]);
    }
    float z = 0.f;
    for (long long c = c_first; c <= c_last; ++c) {
      const float* part = a.partials + ((c + bh) * a.R_pad + r) * W;
      if (part[1] > 0.f) z += expf(part[0] - m) * part[1];
    }
    for (int d = lane; d < D; d += 32) {
      float u = 0.f;
      for (long long c = c_first; c <= c_last; ++c) {
        const float* part = a.partials + ((c + bh) * a.R_pad + r) * W;
        if (part[1] > 0.f) u += expf(part[0] - m) * part[2 + d];
      }
      store_from_f32(a.O, (row_base + r) * D + d, u / z, a.o_dtype);
    }
  }
}

constexpr int kFmRows = 32;       // rows per CTA of the feature-major merge
constexpr int kFmThreads = 256;

__global__ void __launch_bounds__(kFmThreads) merge_fm_kernel(MergeParams mp) {
  extern __shared__ float s_tile[];                // [kFmRows][D + 1], then int pre[B + 1]
  const MergeArgs& a = mp.a;
  const int D = a.D;
  int* s_pre = reinterpret_cast<int*>(s_tile + kFmRows * (D + 1));
  if (threadIdx.x < 32) warp_block_prefix(a.lengths, a.B, a.N_cap, a.BT, s_pre);
  __syncthreads();
  const int H = a.H_kv;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int r0 = blockIdx.y * kFmRows;
  const int rows = min(kFmRows, a.R - r0);
  const long long row_base = (static_cast<long long>(b) * H * a.G + static_cast<long long>(h) * a.G) * a.Lq + r0;
  const int raw_len = a.lengths[b];
  if (h == 0 && blockIdx.y == 0 && threadIdx.x == 0 && (raw_len < 1 || raw_len > a.N_cap))
    record_error(mp.err, KVQ_ERR_LENGTH);
  const int nb = s_pre[b + 1] - s_pre[b];
  if (nb == 0) {
    for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x)
      store_from_f32(a.O, row_base * D + idx, 0.f, a.o_dtype);
    return;
  }
  const CtaRange cr = cta_range(s_pre, a.B, H, a.ctas, 0);
  const long long S = static_cast<long long>(H) * s_pre[b] + static_cast<long long>(h) * nb;
  const long long E = S + nb;
  const long long c_first = S / cr.P, c_last = (E - 1) / cr.P;
  if (c_first == c_last) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const long long slot_floats = static_cast<long long>(D + 2) * a.R_pad;
  if (lane < rows) {
    const int r = r0 + lane;
    float m = -INFINITY;
    for (long long c = c_first; c <= c_last; ++c) {
      const float* part = a.partials + (c + bh) * slot_floats + r;
      if (part[a.R_pad] > 0.f) m = fmaxf(m, part[0]);
    }
    float z = 0.f;
    for (long long c = c_first; c <= c_last; ++c) {
      const float* part = a.partials + (c + bh) * slot_floats + r;
      const float zc = part[a.R_pad];
      if (zc > 0.f) z += expf(part[0] - m) * zc;
    }
    const float inv = 1.f / z;
    for (int d = warp; d < D; d += nwarps) {
      float u = 0.f;
      for (long long c = c_first; c <= c_last; ++c) {
        const float* part = a.partials + (c + bh) * slot_floats + r;
        const float zc = part[a.R_pad];
        if (zc > 0.f) u += expf(part[0] - m) * part[static_cast<long long>(2 + d) * a.R_pad];
      }
      s_tile[lane * (D + 1) + d] = u * inv;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x)
    store_from_f32(a.O, row_base * D + idx, s_tile[(idx / D) * (D + 1) + idx % D], a.o_dtype);
}

}  // namespace

kvq_status launch_merge(const MergeArgs& a, cudaStream_t s) {
  if (a.feature_major) {
    const size_t smem = static_cast<size_t>(kFmRows) * (a.D + 1) * sizeof(float) +
                        static_cast<size_t>(a.B + 1) * sizeof(int);
    const long long bh = static_cast<long long>(a.B) * a.H_kv;
    const int chunks = (a.R + kFmRows - 1) / kFmRows;
    if (bh > 0x7fffffffLL || chunks > 65535) return KVQ_ERR_UNSUPPORTED;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(merge_fm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return KVQ_ERR_UNSUPPORTED;
    MergeParams mp{a, error_word()};
    if (!mp.err) return KVQ_ERR_CUDA;
    merge_fm_kernel<<<dim3(static_cast<unsigned>(bh), static_cast<unsigned>(chunks)), kFmThreads, smem, s>>>(mp);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
  }
  const size_t smem = static_cast<size_t>(a.B + 1) * sizeof(int);
  const long long blocks = static_cast<long long>(a.B) * a.H_kv;
  if (blocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  MergeParams mp{a, error_word()};
  if (!mp.err) return KVQ_ERR_CUDA;
  merge_kernel<<<static_cast<unsigned>(blocks), 128, smem, s>>>(mp);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq

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
// per (b, h), 32-row chunk and 32-feature slice, lane = row so every partial
// read is a coalesced 128-byte line.
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

// Row-major merge: one CTA per (b, h), one thread per (row, feature), so
// the parts' m and z (shared by a row's threads) and then their u values are
// each fetched in one round of independent loads.
__global__ void __launch_bounds__(512) merge_kernel(MergeParams mp) {
  griddep_wait();
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
  const int W = D + 2;
  const long long slot = static_cast<long long>(a.R_pad) * W;
  for (int idx = threadIdx.x; idx < a.R * D; idx += blockDim.x) {
    const int r = idx / D, d = idx % D;
    const float* col = a.partials + (c_first + bh) * slot + static_cast<long long>(r) * W;   // part c: + (c - c_first) * slot
    const int parts = static_cast<int>(c_last - c_first + 1);
    float m = -INFINITY;
#pragma unroll 4
    for (int c = 0; c < parts; ++c) {
      const float zc = col[c * slot + 1], mc = col[c * slot];
      if (zc > 0.f) m = fmaxf(m, mc);
    }
    float z = 0.f, u = 0.f;
#pragma unroll 4
    for (int c = 0; c < parts; ++c) {
      const float zc = col[c * slot + 1], mc = col[c * slot], uc = col[c * slot + 2 + d];
      if (zc > 0.f) {
        const float w = expf(mc - m);
        z = fmaf(w, zc, z);
        u = fmaf(w, uc, u);
      }
    }
    store_from_f32(a.O, (row_base + r) * D + d, u / z, a.o_dtype);
  }
}

constexpr int kFmRows = 32;       // rows per CTA of the feature-major merge
constexpr int kFmCols = 32;       // features per CTA
constexpr int kFmThreads = 128;   // 4 warps x 8 features
constexpr int kFmBatch = 4;       // parts whose weights are held at once

// Feature-major merge: one CTA per (b, h), 32-row chunk and 32-feature
// slice; lane = row, so every read of a part's field is one coalesced
// 128-byte line; warp w owns 8 features.  The weights exp(m_c - m) of up to
// four parts sit in registers and each part's 8 values are loaded together.
__global__ void __launch_bounds__(kFmThreads, 4) merge_fm_kernel(MergeParams mp) {
  griddep_wait();
  extern __shared__ int s_pre[];                   // [B + 1]
  const MergeArgs& a = mp.a;
  const int D = a.D;
  if (threadIdx.x < 32) warp_block_prefix(a.lengths, a.B, a.N_cap, a.BT, s_pre);
  __syncthreads();
  const int H = a.H_kv;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = blockIdx.y * kFmRows + lane;
  const int f0 = blockIdx.z * kFmCols + 8 * warp;
  const long long row = (static_cast<long long>(b) * H * a.G + static_cast<long long>(h) * a.G) * a.Lq + r;
  const int raw_len = a.lengths[b];
  if (h == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0 && (raw_len < 1 || raw_len > a.N_cap))
    record_error(mp.err, KVQ_ERR_LENGTH);
  const bool live = r < a.R && f0 < D;
  const int nb = s_pre[b + 1] - s_pre[b];
  if (nb == 0) {
    if (live)
      for (int j = 0; j < 8 && f0 + j < D; ++j) store_from_f32(a.O, row * D + f0 + j, 0.f, a.o_dtype);
    return;
  }
  const CtaRange cr = cta_range(s_pre, a.B, H, a.ctas, 0);
  const long long S = static_cast<long long>(H) * s_pre[b] + static_cast<long long>(h) * nb;
  const long long E = S + nb;
  const long long c_first = S / cr.P, c_last = (E - 1) / cr.P;
  if (c_first == c_last || !live) return;
  const long long slot_floats = static_cast<long long>(D + 2) * a.R_pad;
  const long long rp = a.R_pad;
  const float* col = a.partials + bh * slot_floats + r;       // part c of this row: col + c * slot_floats
  float m = -INFINITY;
#pragma unroll 4
  for (long long c = c_first; c <= c_last; ++c) {
    const float* part = col + c * slot_floats;
    const float zc = part[rp], mc = part[0];
    if (zc > 0.f) m = fmaxf(m, mc);
  }
  float z = 0.f, u[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) u[j] = 0.f;
  const int nf = min(8, D - f0);
  for (long long cb = c_first; cb <= c_last; cb += kFmBatch) {
    float wgt[kFmBatch], v[kFmBatch][8];
#pragma unroll
    for (int k = 0; k < kFmBatch; ++k) {
      const long long c = min(cb + k, c_last);
      const float* part = col + c * slot_floats;
      const float zc = part[rp], mc = part[0];
      wgt[k] = (cb + k <= c_last && zc > 0.f) ? expf(mc - m) : 0.f;
      z += wgt[k] * (zc > 0.f ? zc : 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[k][j] = j < nf ? part[(2 + f0 + j) * rp] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kFmBatch; ++k)
#pragma unroll
      for (int j = 0; j < 8; ++j) u[j] = fmaf(wgt[k], v[k][j], u[j]);
  }
  const float inv = 1.f / z;
  if (a.o_dtype == KVQ_BF16 && nf == 8) {
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 t = __floats2bfloat162_rn(u[2 * j] * inv, u[2 * j + 1] * inv);
      o[j] = *reinterpret_cast<const uint32_t*>(&t);
    }
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.O) + row * D + f0) = make_uint4(o[0], o[1], o[2], o[3]);
  } else {
    for (int j = 0; j < nf; ++j) store_from_f32(a.O, row * D + f0 + j, u[j] * inv, a.o_dtype);
  }
}

}  // namespace

kvq_status launch_merge(const MergeArgs& a, cudaStream_t s) {
  if (a.feature_major) {
    const size_t smem = static_cast<size_t>(a.B + 1) * sizeof(int);
    const long long bh = static_cast<long long>(a.B) * a.H_kv;
    const int chunks = (a.R + kFmRows - 1) / kFmRows;
    const int slices = (a.D + kFmCols - 1) / kFmCols;
    if (bh > 0x7fffffffLL || chunks > 65535 || slices > 65535 || (a.D % 8) != 0) return KVQ_ERR_UNSUPPORTED;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(merge_fm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return KVQ_ERR_UNSUPPORTED;
    MergeParams mp{a, error_word()};
    if (!mp.err) return KVQ_ERR_CUDA;
    if (launch_pdl(merge_fm_kernel,
                   dim3(static_cast<unsigned>(bh), static_cast<unsigned>(chunks), static_cast<unsigned>(slices)),
                   dim3(kFmThreads), smem, s, mp) != cudaSuccess)
      return KVQ_ERR_CUDA;
    count_launch();
    return KVQ_OK;
  }
  const size_t smem = static_cast<size_t>(a.B + 1) * sizeof(int);
  const long long blocks = static_cast<long long>(a.B) * a.H_kv;
  if (blocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  MergeParams mp{a, error_word()};
  if (!mp.err) return KVQ_ERR_CUDA;
  const long long work = static_cast<long long>(a.R) * a.D;
  const int threads = work >= 512 ? 512 : static_cast<int>((work + 31) / 32 * 32);
  if (launch_pdl(merge_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), smem, s, mp) != cudaSuccess)
    return KVQ_ERR_CUDA;
  count_launch();
  return KVQ_OK;
}

}  // namespace kvq

// Split-KV merge: the (m, z, u) states several workers computed for one (b,
// h) combine with the same rescale rule as the block merge -- m = max of the
// parts, each part scaled by exp(m_part - m) before z and u are summed, a part
// without a valid key (z = 0) skipped -- then O = u / z ("Block KV decoding:
// less workspace, more time", huhohoo.com/en/docs/llm/kv-block-decode-cost,
// section "Do not average independently normalized blocks"; "给长前缀列一张有
// 单位的资源账本", section "FlashAttention为什么不必保存整张热图").
//
// Two layouts of the per-worker partial states (a worker is a CTA, or a warp
// pair of the decode kernel).  Row-major ([slot][row][m, z, u...]), for the
// few-row decode kernels.  Feature-major ([slot][field][row]), for the
// many-row chunk kernel: one CTA per (b, h), 32-row chunk and 32-feature
// slice, lane = row so every partial read is a coalesced 128-byte line.
//
// The parts of (b, h) are the packed-cache workers that covered it (slots
// c + b * H_kv + h for the plan's workers c_first..c_last) and, with a
// recent-token window, the window's state (slot win_slot0 + b * H_kv + h).
// Without a window, a (b, h) that one worker covered whole was already
// written by it and is skipped here.  The merge also owns the sequences with
// no valid key: it records KVQ_ERR_LENGTH and writes zeros.
#include "kvq_internal.cuh"
#include "plan.cuh"

namespace kvq {
namespace {

struct MergeParams {
  MergeArgs a;
  unsigned int* err;
};

// Which parts (b, h) has, and whether the merge writes its rows at all.
struct MergePlan {
  bool zero;              // no valid key: write zero rows
  bool skip;              // one worker covered it whole and wrote it
  long long c_first;      // first packed part's worker
  int parts;              // packed parts (0: none)
  int total;              // packed parts plus the window part
  long long win_slot;     // slot of the window part (valid if total > parts)
};

__device__ __forceinline__ MergePlan merge_plan(const MergeArgs& a, const int* s_pre, int b, int h,
                                                unsigned int* err, bool report) {
  const int H = a.H_kv;
  const int raw = a.lengths[b];
  const int nb = s_pre[b + 1] - s_pre[b];
  int wl = 0;
  bool bad;
  if (a.win_lengths) {
    const int wr = a.win_lengths[b];
    wl = wr < 0 ? 0 : (wr > a.W_cap ? a.W_cap : wr);
    bad = raw < 0 || raw > a.N_cap || wr < 0 || wr > a.W_cap || (nb == 0 && wl == 0);
  } else {
    bad = raw < 1 || raw > a.N_cap || (a.causal && raw < a.Lq);
  }
  if (report && bad) record_error(err, KVQ_ERR_LENGTH);
  MergePlan p{};
  p.zero = nb == 0 && wl == 0;
  p.win_slot = a.win_slot0 + static_cast<long long>(b) * H + h;
  if (nb > 0) {
    const CtaRange cr = cta_range(s_pre, a.B, H, a.ctas, 0);
    const long long S = static_cast<long long>(H) * s_pre[b] + static_cast<long long>(h) * nb;
    const long long E = S + nb;
    p.c_first = S / cr.P;
    p.parts = static_cast<int>((E - 1) / cr.P - p.c_first + 1);
    p.skip = !a.win_lengths && p.parts == 1;
  }
  p.total = p.parts + (wl > 0 ? 1 : 0);
  return p;
}

// Slot of part i of (b, h): a packed worker's, then the window's.
__device__ __forceinline__ long long part_slot(const MergePlan& p, int i, long long bh) {
  return i < p.parts ? p.c_first + i + bh : p.win_slot;
}

// Order-preserving integer keys, so that shared-memory atomicMax finds a
// float maximum.
__device__ __forceinline__ unsigned int order_key(float f) {
  const unsigned int u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_order_key(unsigned int k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Row-major merge for (b, h)s of few parts: one CTA per (b, h).  Pass 1
// spreads the (part, row) pairs over the threads, so each row's largest m
// takes one round of loads; pass 2 gives each thread one (row, feature) and
// walks the parts eight loads deep, weighting each part's z and u by
// exp(m_c - m).
constexpr int kMergeThreads = 512;
constexpr int kMaxMergeRows = 64;   // rows per pass; more rows repeat the passes

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(MergeParams mp) {
  griddep_wait();
  extern __shared__ int s_pre[];                 // [B + 1]
  __shared__ unsigned int s_mkey[kMaxMergeRows];
  const MergeArgs& a = mp.a;
  if (threadIdx.x < 32) warp_block_prefix(a.lengths, a.B, a.N_cap, a.BT, s_pre);
  __syncthreads();
  const int H = a.H_kv;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int D = a.D;
  const long long row_base = (static_cast<long long>(b) * H * a.G + static_cast<long long>(h) * a.G) * a.Lq;
  const MergePlan pl = merge_plan(a, s_pre, b, h, mp.err, h == 0 && threadIdx.x == 0);
  if (pl.zero) {
    for (int idx = threadIdx.x; idx < a.R * D; idx += blockDim.x)
      store_from_f32(a.O, row_base * D + idx, 0.f, a.o_dtype);
    return;
  }
  if (pl.skip) return;
  const int W = D + 2;
  const long long slot = static_cast<long long>(a.R_pad) * W;

  for (int r0 = 0; r0 < a.R; r0 += kMaxMergeRows) {
    const int nr = min(kMaxMergeRows, a.R - r0);
    for (int i = threadIdx.x; i < nr; i += blockDim.x) s_mkey[i] = order_key(-INFINITY);
    __syncthreads();
    // pass 1: each row's largest m over the parts with z > 0
    for (int i = threadIdx.x; i < pl.total * nr; i += blockDim.x) {
      const int c = i / nr, r = r0 + i % nr;
      const float* pr = a.partials + part_slot(pl, c, bh) * slot + static_cast<long long>(r) * W;
      if (pr[1] > 0.f) atomicMax(&s_mkey[r - r0], order_key(pr[0]));
    }
    __syncthreads();
    // pass 2: one (row, feature) per thread
    for (int idx = threadIdx.x; idx < nr * D; idx += blockDim.x) {
      const int r = r0 + idx / D, d = idx % D;
      const float m = from_order_key(s_mkey[r - r0]);
      float z = 0.f, u = 0.f;
#pragma unroll 8
      for (int c = 0; c < pl.total; ++c) {
        const float* pc = a.partials + part_slot(pl, c, bh) * slot + static_cast<long long>(r) * W;
        const float zc = pc[1], mc = pc[0], uc = pc[2 + d];
        if (zc > 0.f) {
          const float w = expf(mc - m);
          z = fmaf(w, zc, z);
          u = fmaf(w, uc, u);
        }
      }
      store_from_f32(a.O, (row_base + r) * D + d, z > 0.f ? u / z : 0.f, a.o_dtype);
    }
    __syncthreads();
  }
}

// Row-major merge for (b, h)s split into many parts (long sequences): one
// CTA per (b, h), row and 32-feature slice; warp w takes parts w, w + 8, ...,
// so the parts are read in one or two rounds of loads.  The parts' largest m
// is found first (pass 1, then over the warps), then each warp sums its
// parts' z and u weighted by exp(m_c - m) (pass 2) and warp 0 adds the eight
// sums.  A lane owns one feature; m and z of a part are one broadcast load.
constexpr int kMW = 8;            // warps = part groups

__global__ void __launch_bounds__(kMW * 32) merge_parts_kernel(MergeParams mp) {
  griddep_wait();
  extern __shared__ int s_pre[];                 // [B + 1]
  __shared__ float s_m[kMW], s_z[kMW], s_u[kMW][32];
  const MergeArgs& a = mp.a;
  if (threadIdx.x < 32) warp_block_prefix(a.lengths, a.B, a.N_cap, a.BT, s_pre);
  __syncthreads();
  const int H = a.H_kv;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int D = a.D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = blockIdx.z;
  const int d = blockIdx.y * 32 + lane;
  const bool live = d < D;
  const long long row = (static_cast<long long>(b) * H * a.G + static_cast<long long>(h) * a.G) * a.Lq + r;
  const MergePlan pl =
      merge_plan(a, s_pre, b, h, mp.err, h == 0 && blockIdx.y == 0 && r == 0 && threadIdx.x == 0);
  if (pl.zero) {
    if (warp == 0 && live) store_from_f32(a.O, row * D + d, 0.f, a.o_dtype);
    return;
  }
  if (pl.skip) return;
  const int W = D + 2;
  const long long slot = static_cast<long long>(a.R_pad) * W;
  const long long roff = static_cast<long long>(r) * W;

  float m = -INFINITY;
#pragma unroll 4
  for (int c = warp; c < pl.total; c += kMW) {
    const float* pc = a.partials + part_slot(pl, c, bh) * slot + roff;
    const float zc = pc[1], mc = pc[0];
    if (zc > 0.f) m = fmaxf(m, mc);
  }
  if (lane == 0) s_m[warp] = m;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kMW; ++w) m = fmaxf(m, s_m[w]);

  float z = 0.f, u = 0.f;
#pragma unroll 4
  for (int c = warp; c < pl.total; c += kMW) {
    const float* pc = a.partials + part_slot(pl, c, bh) * slot + roff;
    const float zc = pc[1], mc = pc[0];
    const float uc = live ? pc[2 + d] : 0.f;
    if (zc > 0.f) {
      const float w = expf(mc - m);
      z = fmaf(w, zc, z);
      u = fmaf(w, uc, u);
    }
  }
  s_u[warp][lane] = u;
  if (lane == 0) s_z[warp] = z;
  __syncthreads();
  if (warp == 0 && live) {
    float zt = 0.f, ut = 0.f;
#pragma unroll
    for (int w = 0; w < kMW; ++w) {
      zt += s_z[w];
      ut += s_u[w][lane];
    }
    store_from_f32(a.O, row * D + d, zt > 0.f ? ut / zt : 0.f, a.o_dtype);
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
  const MergePlan pl =
      merge_plan(a, s_pre, b, h, mp.err, h == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0);
  const bool live = r < a.R && f0 < D;
  if (pl.zero) {
    if (live)
      for (int j = 0; j < 8 && f0 + j < D; ++j) store_from_f32(a.O, row * D + f0 + j, 0.f, a.o_dtype);
    return;
  }
  if (pl.skip || !live) return;
  const long long slot_floats = static_cast<long long>(D + 2) * a.R_pad;
  const long long rp = a.R_pad;
  const float* col = a.partials + r;              // part i of this row: col + part_slot(i) * slot_floats
  float m = -INFINITY;
#pragma unroll 4
  for (int c = 0; c < pl.total; ++c) {
    const float* part = col + part_slot(pl, c, bh) * slot_floats;
    const float zc = part[rp], mc = part[0];
    if (zc > 0.f) m = fmaxf(m, mc);
  }
  float z = 0.f, u[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) u[j] = 0.f;
  const int nf = min(8, D - f0);
  for (int cb = 0; cb < pl.total; cb += kFmBatch) {
    float wgt[kFmBatch], v[kFmBatch][8];
#pragma unroll
    for (int k = 0; k < kFmBatch; ++k) {
      const int c = min(cb + k, pl.total - 1);
      const float* part = col + part_slot(pl, c, bh) * slot_floats;
      const float zc = part[rp], mc = part[0];
      wgt[k] = (cb + k < pl.total && zc > 0.f) ? expf(mc - m) : 0.f;
      z += wgt[k] * (zc > 0.f ? zc : 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[k][j] = j < nf ? part[(2 + f0 + j) * rp] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kFmBatch; ++k)
#pragma unroll
      for (int j = 0; j < 8; ++j) u[j] = fmaf(wgt[k], v[k][j], u[j]);
  }
  const float inv = z > 0.f ? 1.f / z : 0.f;      // z = 0: a causal row with no visible key
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
  const size_t smem = static_cast<size_t>(a.B + 1) * sizeof(int);
  const long long bh = static_cast<long long>(a.B) * a.H_kv;
  if (bh > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  if (smem > 48 * 1024) return KVQ_ERR_UNSUPPORTED;
  MergeParams mp{a, error_word()};
  if (!mp.err) return KVQ_ERR_CUDA;
  cudaError_t le;
  if (a.feature_major) {
    const int chunks = (a.R + kFmRows - 1) / kFmRows;
    const int slices = (a.D + kFmCols - 1) / kFmCols;
    if (chunks > 65535 || slices > 65535 || (a.D % 8) != 0) return KVQ_ERR_UNSUPPORTED;
    le = launch_pdl(merge_fm_kernel, dim3(static_cast<unsigned>(bh), static_cast<unsigned>(chunks),
                                          static_cast<unsigned>(slices)),
                    dim3(kFmThreads), smem, s, mp);
  } else if (a.ctas >= 8 * bh) {
    // on average eight or more workers per (b, h): split the parts over warps
    if (a.R > 65535) return KVQ_ERR_UNSUPPORTED;
    le = launch_pdl(merge_parts_kernel,
                    dim3(static_cast<unsigned>(bh), static_cast<unsigned>((a.D + 31) / 32), static_cast<unsigned>(a.R)),
                    dim3(kMW * 32), smem, s, mp);
  } else {
    const long long work = static_cast<long long>(a.R) * a.D;
    const int threads = work >= kMergeThreads ? kMergeThreads : static_cast<int>((work + 31) / 32 * 32);
    le = launch_pdl(merge_kernel, dim3(static_cast<unsigned>(bh)), dim3(threads), smem, s, mp);
  }
  if (le != cudaSuccess) return KVQ_ERR_CUDA;
  count_launch();
  return KVQ_OK;
}

}  // namespace kvq

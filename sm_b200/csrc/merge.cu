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
// decode and generic kernels: one CTA per (b, h) and row, parts spread over
// its warps.  Feature-major ([slot][field][row]), for the many-row chunk
// kernel: one CTA per (b, h), 32-row chunk and 32-feature slice, lane = row
// so every partial read is a coalesced 128-byte line.  Both load a batch of
// parts (m, z and the thread's u values) before using any of it and fold the
// batch into a running state, so a (b, h) split a few ways costs one round
// trip to memory.
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
  const int raw = __ldcg(a.lengths + b);
  const int nb = s_pre[b + 1] - s_pre[b];
  int wl = 0;
  bool bad;
  if (a.win_lengths) {
    const int wr = __ldcg(a.win_lengths + b);
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
    // nb counts the head's plan slots; its blocks are the first nr of them
    const int nr = seq_blocks(raw, a.N_cap, a.BT);
    const CtaRange cr = cta_range(s_pre, a.B, H, a.ctas, 0);
    const long long S = static_cast<long long>(H) * s_pre[b] + static_cast<long long>(h) * nb;
    const long long E = S + nr;
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

// exp(x) for the merge weights (x <= 0, natural-log units) as one ex2.approx:
// relative error ~2^-22, far inside the attention tolerance; exp(-inf) = 0.
__device__ __forceinline__ float exp_w(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * 1.4426950408889634f));
  return y;
}

// The merge plan of the CTA's (b, h), computed by one thread (after warp 0
// filled s_pre) and shared: its 64-bit divisions run once per CTA.
__device__ __forceinline__ MergePlan shared_plan(const MergeArgs& a, const int* s_pre, int b, int h,
                                                 unsigned int* err, bool report, MergePlan* s_plan) {
  if (threadIdx.x < 32) {
    __syncwarp();
    if (threadIdx.x == 0) *s_plan = merge_plan(a, s_pre, b, h, err, report);
  }
  __syncthreads();
  return *s_plan;
}

// Folds a batch of parts into a running state (M, Z, U[]) with the same
// rule: the batch's largest m over parts that exist (k < n) and hold a key
// (z > 0) becomes the reference if it is larger, the state is scaled by
// exp(M_old - M) and each part adds exp(m_c - M) * (z_c, u_c).  Every load of
// the batch was issued before this runs, so a batch costs one round trip.
template <int PB, int F>
__device__ __forceinline__ void fold_batch(float& M, float& Z, float (&U)[F], const float (&mc)[PB],
                                           const float (&zc)[PB], const float (&uc)[PB][F], int n) {
  float mb = M;
#pragma unroll
  for (int k = 0; k < PB; ++k)
    if (k < n && zc[k] > 0.f) mb = fmaxf(mb, mc[k]);
  if (mb == -INFINITY) return;                       // no key yet
  const float sa = exp_w(M - mb);                    // 0 while M = -inf (Z, U are 0)
  Z *= sa;
#pragma unroll
  for (int j = 0; j < F; ++j) U[j] *= sa;
  M = mb;
#pragma unroll
  for (int k = 0; k < PB; ++k) {
    if (k < n && zc[k] > 0.f) {
      const float w = exp_w(mc[k] - M);
      Z = fmaf(w, zc[k], Z);
#pragma unroll
      for (int j = 0; j < F; ++j) U[j] = fmaf(w, uc[k][j], U[j]);
    }
  }
}

// Row-major merge: one CTA per (b, h) and row, `blockDim.x / 32` warps; lane
// l owns features l + 32 j (D <= 256).  Warp w takes parts w * kRowPB ..
// + kRowPB - 1 of each round of blockDim.x / 32 * kRowPB parts, loading a
// part's m, z and the lane's u values together; the warps' states are then
// combined through shared memory, one feature per thread.
constexpr int kRowPB = 4;         // parts a warp loads per round
constexpr int kRowF = 8;          // features per lane
constexpr int kRowMaxWarps = 8;

__global__ void __launch_bounds__(kRowMaxWarps * 32) merge_rows_kernel(MergeParams mp) {
  extern __shared__ int s_pre[];                 // [B + 1]
  __shared__ float s_m[kRowMaxWarps], s_z[kRowMaxWarps];
  __shared__ float s_u[kRowMaxWarps][256];
  __shared__ MergePlan s_plan;
  const MergeArgs& a = mp.a;
  if (threadIdx.x < 32) warp_block_prefix(a.lengths, a.B, a.N_cap, a.BT, s_pre, true, a.extra_slots);
  const int H = a.H_kv;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int D = a.D;
  const int r = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const long long row = (static_cast<long long>(b) * H * a.G + static_cast<long long>(h) * a.G) * a.Lq + r;
  const MergePlan pl = shared_plan(a, s_pre, b, h, mp.err, h == 0 && r == 0, &s_plan);
  griddep_wait();                                // the plan ran beside the kernel before; now its parts
  if (pl.zero) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) store_from_f32(a.O, row * D + d, 0.f, a.o_dtype);
    return;
  }
  if (pl.skip) return;
  const long long slot = static_cast<long long>(a.R_pad) * (D + 2);
  const long long roff = static_cast<long long>(r) * (D + 2);

  float M = -INFINITY, Z = 0.f, U[kRowF];
#pragma unroll
  for (int j = 0; j < kRowF; ++j) U[j] = 0.f;
  for (int base = warp * kRowPB; base < pl.total; base += nw * kRowPB) {
    float mc[kRowPB], zc[kRowPB], uc[kRowPB][kRowF];
#pragma unroll
    for (int k = 0; k < kRowPB; ++k) {
      const int c = min(base + k, pl.total - 1);   // past the last part: reload it, masked below
      const float* pc = a.partials + part_slot(pl, c, bh) * slot + roff;
      mc[k] = pc[0];
      zc[k] = pc[1];
#pragma unroll
      for (int j = 0; j < kRowF; ++j) {
        const int d = lane + 32 * j;
        uc[k][j] = d < D ? pc[2 + d] : 0.f;
      }
    }
    fold_batch<kRowPB, kRowF>(M, Z, U, mc, zc, uc, pl.total - base);
  }
  if (lane == 0) {
    s_m[warp] = M;
    s_z[warp] = Z;
  }
#pragma unroll
  for (int j = 0; j < kRowF; ++j) {
    const int d = lane + 32 * j;
    if (d < D) s_u[warp][d] = U[j];
  }
  __syncthreads();
  float Mt = -INFINITY;
  for (int w = 0; w < nw; ++w)
    if (s_z[w] > 0.f) Mt = fmaxf(Mt, s_m[w]);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float z = 0.f, u = 0.f;
    for (int w = 0; w < nw; ++w) {
      if (s_z[w] > 0.f) {
        const float e = exp_w(s_m[w] - Mt);
        z = fmaf(e, s_z[w], z);
        u = fmaf(e, s_u[w][d], u);
      }
    }
    store_from_f32(a.O, row * D + d, z > 0.f ? u / z : 0.f, a.o_dtype);   // z = 0: a row with no key
  }
}

// Feature-major merge: one CTA per (b, h), 32-row chunk and 32-feature
// slice; lane = row, so each field read of a part is one coalesced 128-byte
// line, and a chunk's fields are consecutive lines (a slice's 32 features
// are 4 KB in one run); warp w owns features 4w .. 4w + 3.  A thread loads
// m, z and its four u values of kFmPB parts per round; small rounds keep
// the registers low enough for five CTAs per SM, so the grid runs in fewer
// waves (each wave pays the prefix and plan chain once).
constexpr int kFmRows = 32;       // rows per CTA
constexpr int kFmF = 4;           // features per thread
constexpr int kFmWarps = 8;       // 8 x 4 = 32 features per CTA
constexpr int kFmPB = 4;          // parts per round (two rounds for the usual 5-6)

// DC: the head dimension when it is fixed at compile time (128, the chunk
// kernel's: the field offsets fold into constants, chunk attend -2 us), else
// 0.  The row-major merge stays on the runtime D: fixed, it measured 2 us
// slower on the decode workload.
template <int DC>
__global__ void __launch_bounds__(kFmWarps * 32, 5) merge_fm_kernel(MergeParams mp) {
  extern __shared__ int s_pre[];                   // [B + 1]
  __shared__ MergePlan s_plan;
  const MergeArgs& a = mp.a;
  const int D = DC ? DC : a.D;
  if (threadIdx.x < 32) warp_block_prefix(a.lengths, a.B, a.N_cap, a.BT, s_pre, true, a.extra_slots);
  const int H = a.H_kv;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = blockIdx.y * kFmRows + lane;
  const int f0 = blockIdx.z * (kFmWarps * kFmF) + kFmF * warp;
  const long long row = (static_cast<long long>(b) * H * a.G + static_cast<long long>(h) * a.G) * a.Lq + r;
  const MergePlan pl = shared_plan(a, s_pre, b, h, mp.err, h == 0 && blockIdx.y == 0 && blockIdx.z == 0, &s_plan);
  griddep_wait();                                  // the plan ran beside the kernel before; now its parts
  const bool live = r < a.R && f0 < D;
  const int nf = min(kFmF, D - f0);
  if (pl.zero) {
    if (live)
      for (int j = 0; j < nf; ++j) store_from_f32(a.O, row * D + f0 + j, 0.f, a.o_dtype);
    return;
  }
  if (pl.skip || !live) return;
  const long long slot_floats = static_cast<long long>(D + 2) * a.R_pad;
  // field f of row r within a slot: (r / 32) * (D + 2) * 32 + f * 32 + r % 32
  const float* col = a.partials + static_cast<long long>(r >> 5) * (D + 2) * 32 + (r & 31);
  float M = -INFINITY, Z = 0.f, U[kFmF];
#pragma unroll
  for (int j = 0; j < kFmF; ++j) U[j] = 0.f;
  for (int base = 0; base < pl.total; base += kFmPB) {
    float mc[kFmPB], zc[kFmPB], uc[kFmPB][kFmF];
#pragma unroll
    for (int k = 0; k < kFmPB; ++k) {
      const int c = min(base + k, pl.total - 1);
      const float* part = col + part_slot(pl, c, bh) * slot_floats;
      mc[k] = part[0];
      zc[k] = part[32];
#pragma unroll
      for (int j = 0; j < kFmF; ++j) uc[k][j] = j < nf ? part[(2 + f0 + j) * 32] : 0.f;
    }
    fold_batch<kFmPB, kFmF>(M, Z, U, mc, zc, uc, pl.total - base);
  }
  const float inv = Z > 0.f ? 1.f / Z : 0.f;      // Z = 0: a causal row with no visible key
  if (a.o_dtype == KVQ_BF16 && nf == kFmF) {
    const __nv_bfloat162 t0 = __floats2bfloat162_rn(U[0] * inv, U[1] * inv);
    const __nv_bfloat162 t1 = __floats2bfloat162_rn(U[2] * inv, U[3] * inv);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.O) + row * D + f0) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&t0), *reinterpret_cast<const uint32_t*>(&t1));
  } else {
    for (int j = 0; j < nf; ++j) store_from_f32(a.O, row * D + f0 + j, U[j] * inv, a.o_dtype);
  }
}

}  // namespace

kvq_status launch_merge(const MergeArgs& a, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(a.B + 1) * sizeof(int);
  const long long bh = static_cast<long long>(a.B) * a.H_kv;
  if (bh > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  if (smem > 48 * 1024 || a.D > 256 || a.D < 1) return KVQ_ERR_UNSUPPORTED;
  MergeParams mp{a, error_word()};
  if (!mp.err) return KVQ_ERR_CUDA;
  cudaError_t le;
  if (a.feature_major) {
    const int chunks = (a.R + kFmRows - 1) / kFmRows;
    const int slices = (a.D + kFmWarps * kFmF - 1) / (kFmWarps * kFmF);
    if (chunks > 65535 || slices > 65535 || (a.D % 8) != 0 || (a.R_pad % 32) != 0) return KVQ_ERR_UNSUPPORTED;
    le = launch_pdl(a.D == 128 ? merge_fm_kernel<128> : merge_fm_kernel<0>, dim3(static_cast<unsigned>(bh), static_cast<unsigned>(chunks),
                                          static_cast<unsigned>(slices)),
                    dim3(kFmWarps * 32), smem, s, mp);
  } else {
    // warps per row: enough for the workers' average share of a (b, h) (plus
    // the ragged ends and a window part) in one round
    if (a.R > 65535) return KVQ_ERR_UNSUPPORTED;
    const long long parts = (static_cast<long long>(a.ctas) + bh - 1) / bh + 2;
    const long long nw = std::min<long long>(kRowMaxWarps, std::max<long long>(1, (parts + kRowPB - 1) / kRowPB));
    le = launch_pdl(merge_rows_kernel, dim3(static_cast<unsigned>(bh), static_cast<unsigned>(a.R)),
                    dim3(static_cast<unsigned>(nw * 32)), smem, s, mp);
  }
  if (le != cudaSuccess) return KVQ_ERR_CUDA;
  count_launch();
  return KVQ_OK;
}

}  // namespace kvq

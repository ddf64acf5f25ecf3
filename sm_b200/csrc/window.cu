// Partial attention state over the recent-token window: the unquantized keys
// that follow each sequence's packed tokens (kvq_attend_window).
//
// The pages leave the window as their next study: keep the packed format and
// spend a limited high-precision budget on the most recent tokens
// ("KV分组打包：4-bit到底省了多少？", section "小练习与常见错误", last
// paragraph).  Each query row's softmax runs over the packed keys and the
// window keys together; this kernel computes the window's share as one more
// (m, z, u) state -- m the largest score, z = sum exp(s - m), u = sum exp(s -
// m) v -- which the split merge folds in with the block rule ("Block KV
// decoding: less workspace, more time", huhohoo.com/en/docs/llm/
// kv-block-decode-cost, section "Do not average independently normalized
// blocks").
//
// One CTA of eight warps per (b, h_kv, pass), a pass being up to 32 of the
// head's query rows (RP rows); window tokens 32 at a time are staged in
// shared memory as f32, their scores computed, and the rows' running
// (m, z, u) updated with the same rule.  Every index is warp-strided -- warp w owns rows (or tokens)
// w, w + 8, w + 16, w + 24 and lane l owns features l, l + 32, ... -- so no
// division runs per element, and a pass's Q rows go out in one batch of loads
// with the first tile's K and V rows.  The kernel reads only the call's inputs
// and writes its own slots, so it runs beside the packed-cache kernel before
// it and joins that kernel's grid only at its end.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWT = 32;          // window tokens per tile
constexpr int kWR = 32;          // largest rows per pass
constexpr int kWThreads = 256;
constexpr int kWWarps = kWThreads / 32;
static_assert(kWT == 32, "the softmax of a tile runs one token per lane");
static_assert(kWT == 4 * kWWarps && kWR == 4 * kWWarps, "a warp stages four rows of a tile");

struct WindowParams {
  WindowArgs a;
};

int rows_per_pass(const WindowArgs& a) {
  const int R = a.G * a.Lq;
  return R < kWR ? (R < 1 ? 1 : R) : kWR;
}

// shared memory: q [RP][D], u [RP][D], K and V tiles [kWT][D + 1],
// p [RP][kWT], m, z, alpha [RP]
size_t window_smem(int D, int RP) {
  return sizeof(float) * (2 * static_cast<size_t>(RP) * D + 2 * static_cast<size_t>(kWT) * (D + 1) +
                          static_cast<size_t>(RP) * kWT + 3 * static_cast<size_t>(RP));
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// rows warp + 8k (k < 4) of the row-major [.][D] array at p, feature
// lane + 32j in v[k][j]; rows at or past n_live and features past D read 0.
// The reads go to the L2 (ld.global.cg): the kernel reads its inputs before
// its grid-dependency wait.
template <int JMAX, typename T>
__device__ __forceinline__ void load_rows(float (&v)[4][JMAX], const T* p, int D, int n_live, int warp, int lane) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = warp + kWWarps * k;
#pragma unroll
    for (int j = 0; j < JMAX; ++j) {
      const int d = lane + 32 * j;
      v[k][j] = (r < n_live && d < D) ? to_f32(__ldcg(p + static_cast<long long>(r) * D + d)) : 0.f;
    }
  }
}

template <int JMAX>
__device__ __forceinline__ void load_rows_any(float (&v)[4][JMAX], const void* p, int dtype, long long off, int D,
                                              int n_live, int warp, int lane) {
  if (dtype == KVQ_F32) load_rows<JMAX>(v, static_cast<const float*>(p) + off, D, n_live, warp, lane);
  else load_rows<JMAX>(v, static_cast<const __nv_bfloat16*>(p) + off, D, n_live, warp, lane);
}

// v[k][j] to s[(warp + 8k) * stride + lane + 32j] for the rows below n_rows
template <int JMAX>
__device__ __forceinline__ void store_rows(float* s, int stride, const float (&v)[4][JMAX], int D, int n_rows,
                                           int warp, int lane) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = warp + kWWarps * k;
#pragma unroll
    for (int j = 0; j < JMAX; ++j) {
      const int d = lane + 32 * j;
      if (r < n_rows && d < D) s[r * stride + d] = v[k][j];
    }
  }
}

// Scores of a tile, s_p[r][t] = scale * q_r . k_t, for a pass of at most 8
// rows: item (r, t) per thread; when there are fewer items than threads,
// `parts` adjacent lanes split an item's dot product (features part, part +
// parts, ...) and add with shuffles.
__device__ __forceinline__ void scores_few_rows(float* s_p, const float* s_q, const float* s_k, int rows, int nt,
                                                int D, int DS, float scale) {
  const int items = rows * kWT;
  const int parts = items * 2 > kWThreads ? 1 : items * 4 > kWThreads ? 2 : items * 8 > kWThreads ? 4 : 8;
  const int per = kWThreads / parts;                 // items per sweep
  for (int base = 0; base < items; base += per) {
    const int it = base + static_cast<int>(threadIdx.x) / parts;
    const int pt = static_cast<int>(threadIdx.x) % parts;
    const int r = it / kWT, t = it - r * kWT;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (it < items && t < nt) {
      const float* qr = s_q + r * D;
      const float* kr = s_k + t * DS;
      int d = pt;
      for (; d + 3 * parts < D; d += 4 * parts) {
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = fmaf(qr[d + j * parts], kr[d + j * parts], acc[j]);
      }
      for (; d < D; d += parts) acc[0] = fmaf(qr[d], kr[d], acc[0]);
    }
    float sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    for (int o = 1; o < parts; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (it < items && pt == 0) s_p[r * kWT + t] = t < nt ? sum * scale : -INFINITY;
  }
}

// The same for a pass of more rows: warp w takes rows 4w .. 4w + 3, lane l
// token l, so a K element read once serves four rows (the Q elements are
// broadcast reads, four features at a time when D is a multiple of 4).
__device__ __forceinline__ void scores_many_rows(float* s_p, const float* s_q, const float* s_k, int rows, int nt,
                                                 int D, int DS, float scale, int warp, int lane) {
  const int rb = 4 * warp;
  if (rb >= rows) return;
  const float* q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = s_q + min(rb + i, rows - 1) * D;
  const float* kr = s_k + lane * DS;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int d = 0;
  if ((D & 3) == 0) {
#pragma unroll 8
    for (; d < D; d += 4) {
      const float k0 = kr[d], k1 = kr[d + 1], k2 = kr[d + 2], k3 = kr[d + 3];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 qv = *reinterpret_cast<const float4*>(q[i] + d);
        acc[i] = fmaf(qv.x, k0, acc[i]);
        acc[i] = fmaf(qv.y, k1, acc[i]);
        acc[i] = fmaf(qv.z, k2, acc[i]);
        acc[i] = fmaf(qv.w, k3, acc[i]);
      }
    }
  }
  for (; d < D; ++d) {
    const float kv = kr[d];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = fmaf(q[i][d], kv, acc[i]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (rb + i < rows) s_p[(rb + i) * kWT + lane] = lane < nt ? acc[i] * scale : -INFINITY;
}

// u = alpha u + p V over the tile's tokens (the first tile starts u from
// zero), for a pass of at most 8 rows: a warp per (row, 32 features), four
// chains over the tokens.
__device__ __forceinline__ void pv_few_rows(float* s_u, const float* s_p, const float* s_v, const float* s_a,
                                            bool first, int rows, int nt, int D, int DS, int warp, int lane) {
  const int nj = (D + 31) >> 5;
  for (int item = warp; item < rows * nj; item += kWWarps) {
    const int r = item / nj, j = item - r * nj;
    const int d = lane + 32 * j;
    if (d < D) {
      const float* pr = s_p + r * kWT;
      const float* vc = s_v + d;
      float c0 = first ? 0.f : s_a[r] * s_u[r * D + d], c1 = 0.f, c2 = 0.f, c3 = 0.f;
      int t = 0;
      for (; t + 4 <= nt; t += 4) {
        c0 = fmaf(pr[t], vc[t * DS], c0);
        c1 = fmaf(pr[t + 1], vc[(t + 1) * DS], c1);
        c2 = fmaf(pr[t + 2], vc[(t + 2) * DS], c2);
        c3 = fmaf(pr[t + 3], vc[(t + 3) * DS], c3);
      }
      for (; t < nt; ++t) c0 = fmaf(pr[t], vc[t * DS], c0);
      s_u[r * D + d] = (c0 + c1) + (c2 + c3);
    }
  }
}

// The same for a pass of more rows: warp w takes rows 4w .. 4w + 3, lane l
// features l, l + 32, ..., so a V element read once serves four rows.
template <int JMAX>
__device__ __forceinline__ void pv_many_rows(float* s_u, const float* s_p, const float* s_v, const float* s_a,
                                             bool first, int rows, int nt, int D, int DS, int warp, int lane) {
  const int rb = 4 * warp;
  if (rb >= rows) return;
  float acc[4][JMAX];
  int pr[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    pr[i] = min(rb + i, rows - 1);
    const float al = first ? 0.f : s_a[pr[i]];
#pragma unroll
    for (int j = 0; j < JMAX; ++j) {
      const int d = lane + 32 * j;
      acc[i][j] = (first || d >= D) ? 0.f : al * s_u[pr[i] * D + d];
    }
  }
  for (int t = 0; t < nt; ++t) {
    float p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = s_p[pr[i] * kWT + t];
#pragma unroll
    for (int j = 0; j < JMAX; ++j) {
      const int d = lane + 32 * j;
      const float v = s_v[t * DS + min(d, D)];      // column D is the row's padding
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(p[i], v, acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < JMAX; ++j) {
      const int d = lane + 32 * j;
      if (rb + i < rows && d < D) s_u[(rb + i) * D + d] = acc[i][j];
    }
}

// JMAX: features per lane, D <= 32 * JMAX; DC: D when it is fixed at compile
// time (128), else 0.  One CTA per (b, h_kv, pass of
// RP rows); the body is a grid-stride loop over the passes, which at this
// grid runs once (the loop form measured 4 to 8 us faster per step than the
// same body without it on the decode workload's window).  Two CTAs per SM:
// the grid of a decode step, B * H_kv CTAs, then fits in one wave.
template <int JMAX, int DC>
__global__ void __launch_bounds__(kWThreads, 2) window_kernel(WindowParams wp) {
  griddep_release();
  const WindowArgs& a = wp.a;
  extern __shared__ float sm[];
  const int D = DC ? DC : a.D, DS = D + 1;
  const int R = a.G * a.Lq;
  const int RP = R < kWR ? R : kWR;
  if (RP < 1) {
    griddep_join();
    return;
  }
  const int passes = (R + RP - 1) / RP;
  float* s_q = sm;                       // [RP][D]
  float* s_u = s_q + RP * D;             // [RP][D]
  float* s_k = s_u + RP * D;             // [kWT][DS]
  float* s_v = s_k + kWT * DS;           // [kWT][DS]
  float* s_p = s_v + kWT * DS;           // [RP][kWT]
  float* s_m = s_p + RP * kWT;
  float* s_z = s_m + RP;
  float* s_a = s_z + RP;

  const int bh = static_cast<int>(blockIdx.x) / passes;
  const int r_first = (static_cast<int>(blockIdx.x) - bh * passes) * RP;
  const int b = bh / a.H_kv, h = bh % a.H_kv;
  const int raw = __ldcg(a.win_lengths + b);
  const int wl = raw < 0 ? 0 : (raw > a.W_cap ? a.W_cap : raw);
  const long long row_base = (static_cast<long long>(b) * a.H_kv * a.G + static_cast<long long>(h) * a.G) * a.Lq;
  const long long win_base = static_cast<long long>(bh) * a.W_cap * D;
  float* slot = a.partials + (a.slot0 + bh) * a.slot_stride;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r0 = r_first; r0 < R; r0 += RP * passes) {
    const int rows = min(RP, R - r0);
    const bool many = rows > 8;
    {
      // the pass's Q rows and the window's first tile, all loads issued
      // before any store
      float qv[4][JMAX], kv[4][JMAX], vv[4][JMAX];
      const int nt0 = min(kWT, wl);
      load_rows_any<JMAX>(qv, a.Q, a.q_dtype, (row_base + r0) * D, D, rows, warp, lane);
      load_rows_any<JMAX>(kv, a.K_win, a.win_dtype, win_base, D, nt0, warp, lane);
      load_rows_any<JMAX>(vv, a.V_win, a.win_dtype, win_base, D, nt0, warp, lane);
      store_rows<JMAX>(s_q, D, qv, D, rows, warp, lane);
      store_rows<JMAX>(s_k, DS, kv, D, kWT, warp, lane);
      store_rows<JMAX>(s_v, DS, vv, D, kWT, warp, lane);
    }
    if (threadIdx.x < RP) {
      s_m[threadIdx.x] = -INFINITY;
      s_z[threadIdx.x] = 0.f;
    }
    __syncthreads();
    for (int t0 = 0; t0 < wl; t0 += kWT) {
      const int nt = min(kWT, wl - t0);
      if (t0 > 0) {
        float kv[4][JMAX], vv[4][JMAX];
        const long long off = win_base + static_cast<long long>(t0) * D;
        load_rows_any<JMAX>(kv, a.K_win, a.win_dtype, off, D, nt, warp, lane);
        load_rows_any<JMAX>(vv, a.V_win, a.win_dtype, off, D, nt, warp, lane);
        store_rows<JMAX>(s_k, DS, kv, D, kWT, warp, lane);
        store_rows<JMAX>(s_v, DS, vv, D, kWT, warp, lane);
        __syncthreads();
      }
      if (many) scores_many_rows(s_p, s_q, s_k, rows, nt, D, DS, a.scale, warp, lane);
      else scores_few_rows(s_p, s_q, s_k, rows, nt, D, DS, a.scale);
      __syncthreads();
      // the block rule: m_new = max(m, tile max), alpha = exp(m - m_new);
      // a warp per row, lane = token of the tile
      for (int r = warp; r < rows; r += kWWarps) {
        const float sc = s_p[r * kWT + lane];          // -inf past the tile's tokens
        float mb = sc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
        const float mo = s_m[r];
        const float mn = fmaxf(mo, mb);
        const float e = lane < nt ? expf(sc - mn) : 0.f;
        float zs = e;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
        s_p[r * kWT + lane] = e;
        __syncwarp();
        if (lane == 0) {
          const float al = mo == -INFINITY ? 0.f : expf(mo - mn);
          s_z[r] = al * s_z[r] + zs;
          s_m[r] = mn;
          s_a[r] = al;
        }
      }
      __syncthreads();
      if (many) pv_many_rows<JMAX>(s_u, s_p, s_v, s_a, t0 == 0, rows, nt, D, DS, warp, lane);
      else pv_few_rows(s_u, s_p, s_v, s_a, t0 == 0, rows, nt, D, DS, warp, lane);
      __syncthreads();
    }
    // the rows' window states; an empty window leaves m = -inf, z = 0, u = 0
    for (int r = warp; r < rows; r += kWWarps) {
      const long long rr = r0 + r;
      float* dst = slot + (rr >> 5) * a.row_chunk_stride + (rr & 31) * a.row_stride;
      for (int f = lane; f < D + 2; f += 32) {
        const float v = f == 0 ? s_m[r] : (f == 1 ? s_z[r] : (wl > 0 ? s_u[r * D + f - 2] : 0.f));
        dst[static_cast<long long>(f) * a.field_stride] = v;
      }
    }
    __syncthreads();
  }
  griddep_join();
}

}  // namespace

kvq_status add_window(const AttendArgs& a, float* partials, long long slot0, long long slot_stride,
                      long long row_stride, long long row_chunk_stride, long long field_stride, MergeArgs* m,
                      cudaStream_t s) {
  if (!a.win_lengths) return KVQ_OK;
  WindowArgs w{};
  w.Q = a.Q;
  w.q_dtype = a.q_dtype;
  w.K_win = a.K_win;
  w.V_win = a.V_win;
  w.win_dtype = a.win_dtype;
  w.win_lengths = a.win_lengths;
  w.W_cap = a.W_cap;
  w.B = a.g.B;
  w.H_kv = a.g.H_kv;
  w.G = a.H_q / a.g.H_kv;
  w.Lq = a.Lq;
  w.D = a.g.D;
  w.scale = a.scale;
  w.partials = partials;
  w.slot0 = slot0;
  w.slot_stride = slot_stride;
  w.row_stride = row_stride;
  w.row_chunk_stride = row_chunk_stride;
  w.field_stride = field_stride;
  const kvq_status st = launch_window(w, s);
  if (st != KVQ_OK) return st;
  m->win_lengths = a.win_lengths;
  m->W_cap = a.W_cap;
  m->win_slot0 = slot0;
  return KVQ_OK;
}

kvq_status launch_window(const WindowArgs& w, cudaStream_t s) {
  const int RP = rows_per_pass(w);
  const long long passes = (static_cast<long long>(w.G) * w.Lq + RP - 1) / RP;
  const long long blocks = static_cast<long long>(w.B) * w.H_kv * (passes < 1 ? 1 : passes);
  if (blocks > 0x7fffffffLL || w.D > 256 || w.D < 1) return KVQ_ERR_UNSUPPORTED;
  const size_t smem = window_smem(w.D, RP);
  // D = 128 as a compile-time constant: the score loops unroll fully
  auto kernel = w.D == 128 ? window_kernel<4, 128>
                           : (w.D <= 64 ? window_kernel<2, 0> : (w.D <= 128 ? window_kernel<4, 0> : window_kernel<8, 0>));
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kernel), smem)) return KVQ_ERR_CUDA;
  WindowParams p{w};
  if (launch_pdl(kernel, dim3(static_cast<unsigned>(blocks)), dim3(kWThreads), smem, s, p) != cudaSuccess)
    return KVQ_ERR_CUDA;
  count_launch();
  return KVQ_OK;
}

}  // namespace kvq

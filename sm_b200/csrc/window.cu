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
// One CTA per (b, h_kv).  Rows are taken 32 at a time; window tokens 32 at a
// time are staged in shared memory as f32, their scores computed, and the
// rows' running (m, z, u) updated with the same rule.  The window is short
// (a few groups at most), so this is a small kernel next to the packed path.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWT = 32;          // window tokens per tile
constexpr int kWR = 32;          // rows per pass
constexpr int kWThreads = 256;
static_assert(kWT == 32, "the softmax of a tile runs one token per lane");

struct WindowParams {
  WindowArgs a;
};

// shared memory: q [kWR][D], u [kWR][D], K and V tiles [kWT][D + 1],
// p [kWR][kWT], m, z, alpha [kWR]
size_t window_smem(int D) {
  return sizeof(float) * (2 * static_cast<size_t>(kWR) * D + 2 * static_cast<size_t>(kWT) * (D + 1) +
                          kWR * kWT + 3 * kWR);
}

__global__ void __launch_bounds__(kWThreads) window_kernel(WindowParams wp) {
  griddep_wait();
  const WindowArgs& a = wp.a;
  extern __shared__ float sm[];
  const int D = a.D, DS = D + 1;
  float* s_q = sm;                       // [kWR][D]
  float* s_u = s_q + kWR * D;            // [kWR][D]
  float* s_k = s_u + kWR * D;            // [kWT][DS]
  float* s_v = s_k + kWT * DS;           // [kWT][DS]
  float* s_p = s_v + kWT * DS;           // [kWR][kWT]
  float* s_m = s_p + kWR * kWT;
  float* s_z = s_m + kWR;
  float* s_a = s_z + kWR;

  const int bh = blockIdx.x;
  const int b = bh / a.H_kv, h = bh % a.H_kv;
  const int R = a.G * a.Lq;
  const int raw = a.win_lengths[b];
  const int wl = raw < 0 ? 0 : (raw > a.W_cap ? a.W_cap : raw);
  const long long row_base = (static_cast<long long>(b) * a.H_kv * a.G + static_cast<long long>(h) * a.G) * a.Lq;
  const long long win_base = static_cast<long long>(bh) * a.W_cap * D;
  float* slot = a.partials + (a.slot0 + bh) * a.slot_stride;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r0 = 0; r0 < R; r0 += kWR) {
    const int rows = min(kWR, R - r0);
    for (int i0 = threadIdx.x; i0 < rows * D; i0 += kWThreads * 8) {
      float qv[8];                                     // eight loads in flight per thread
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kWThreads;
        qv[u] = i < rows * D ? load_as_f32(a.Q, (row_base + r0) * D + i, a.q_dtype) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (i0 + u * kWThreads < rows * D) s_q[i0 + u * kWThreads] = qv[u];
    }
    for (int i = threadIdx.x; i < kWR * D; i += blockDim.x) s_u[i] = 0.f;
    if (threadIdx.x < kWR) {
      s_m[threadIdx.x] = -INFINITY;
      s_z[threadIdx.x] = 0.f;
    }
    __syncthreads();
    for (int t0 = 0; t0 < wl; t0 += kWT) {
      const int nt = min(kWT, wl - t0);
      // the tile's K and V rows, all of a thread's loads issued before any store
      for (int i0 = threadIdx.x; i0 < kWT * D; i0 += kWThreads * 8) {
        float kv[8], vv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kWThreads;
          const bool live = i < nt * D;
          const long long e = win_base + static_cast<long long>(t0) * D + i;
          kv[u] = live ? load_as_f32(a.K_win, e, a.win_dtype) : 0.f;
          vv[u] = live ? load_as_f32(a.V_win, e, a.win_dtype) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kWThreads;
          if (i < kWT * D) {
            const int t = i / D, d = i - t * D;
            s_k[t * DS + d] = kv[u];
            s_v[t * DS + d] = vv[u];
          }
        }
      }
      __syncthreads();
      // scores of the tile
      for (int i = threadIdx.x; i < kWR * kWT; i += blockDim.x) {
        const int r = i / kWT, t = i - r * kWT;
        float sc = -INFINITY;
        if (r < rows && t < nt) {
          float acc = 0.f;
          for (int d = 0; d < D; ++d) acc = fmaf(s_q[r * D + d], s_k[t * DS + d], acc);
          sc = acc * a.scale;
        }
        s_p[i] = sc;
      }
      __syncthreads();
      // the block rule: m_new = max(m, tile max), alpha = exp(m - m_new);
      // a warp per row, lane = token of the tile
      for (int r = warp; r < rows; r += kWThreads / 32) {
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
      for (int i = threadIdx.x; i < rows * D; i += blockDim.x) {
        const int r = i / D, d = i - r * D;
        float acc = s_a[r] * s_u[i];
        for (int t = 0; t < nt; ++t) acc = fmaf(s_p[r * kWT + t], s_v[t * DS + d], acc);
        s_u[i] = acc;
      }
      __syncthreads();
    }
    // the rows' window states; an empty window leaves m = -inf, z = 0
    for (int i = threadIdx.x; i < rows * (D + 2); i += blockDim.x) {
      const int r = i / (D + 2), f = i - r * (D + 2);
      const float v = f == 0 ? s_m[r] : (f == 1 ? s_z[r] : s_u[r * D + f - 2]);
      const long long rr = r0 + r;
      slot[(rr >> 5) * a.row_chunk_stride + (rr & 31) * a.row_stride + static_cast<long long>(f) * a.field_stride] = v;
    }
    __syncthreads();
  }
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
  const long long blocks = static_cast<long long>(w.B) * w.H_kv;
  if (blocks > 0x7fffffffLL || w.D > 256 || w.D < 1) return KVQ_ERR_UNSUPPORTED;
  const size_t smem = window_smem(w.D);
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(window_kernel), smem)) return KVQ_ERR_CUDA;
  WindowParams p{w};
  if (launch_pdl(window_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kWThreads), smem, s, p) != cudaSuccess)
    return KVQ_ERR_CUDA;
  count_launch();
  return KVQ_OK;
}

}  // namespace kvq

// Generic packed-KV attention: any width D <= 256, 4- or 8-bit codes, any
// even group, any GQA ratio and any number of query rows.  Correctness path
// for the small and odd shapes; the tuned kernels take the large ones.
//
// Per block of 32 tokens the CTA decodes K and V into shared memory as
// float32 -- (code - qmax) * scale, the same float32 operations a NumPy
// decode performs -- scores its query rows against them and folds the block
// into the running (m, z, u) with the block rule ("Block KV decoding: less
// workspace, more time", huhohoo.com/en/docs/llm/kv-block-decode-cost,
// section "Do not average independently normalized blocks").  Nothing
// decoded leaves shared memory.
#include "kvq_internal.cuh"
#include "plan.cuh"

namespace kvq {
namespace {

constexpr int kBT = 32;        // tokens per block
constexpr int kRT = 16;        // query rows per CTA (row tile)
constexpr int kThreads = 256;

struct GenericParams {
  const void* Q;
  int q_dtype;
  const uint8_t* k_codes;
  const float* k_scales;
  const uint8_t* v_codes;
  const float* v_scales;
  const int32_t* lengths;
  int bits, group, B, H, N_cap, D, Dp;
  long long k_codes_head, k_scales_head, v_codes_head, v_scales_head;
  int G, Lq, R, n_rt;          // q heads per kv head, rows per query head, rows per (b,h), row tiles
  float scale;
  void* O;
  float* partials;             // [slots][n_rt*kRT][D + 2]
  int ctas;
  int force_partial;           // a window follows: no CTA writes output rows
  int causal;                  // query i of Lq reads keys [0, len - Lq + i] only
};

__device__ __forceinline__ int code_at(const uint8_t* codes, long long flat, int bits) {
  if (bits == 8) return codes[flat];
  const unsigned b = codes[flat >> 1];
  return (flat & 1) ? static_cast<int>(b >> 4) : static_cast<int>(b & 15u);
}

size_t smem_bytes(int D, int B) {
  return (static_cast<size_t>(2 * kBT * (D + 1) + 2 * kRT * D + kRT * kBT + 3 * kRT) * sizeof(float)) +
         static_cast<size_t>(B + 1) * sizeof(int);
}

__global__ void __launch_bounds__(kThreads) attend_generic_kernel(GenericParams p) {
  griddep_wait();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int D = p.D;
  const int DS = D + 1;                               // padded row stride: no bank conflicts
  float* s_k = reinterpret_cast<float*>(smem_raw);   // [kBT][DS]
  float* s_v = s_k + kBT * DS;                        // [kBT][DS]
  float* s_q = s_v + kBT * DS;                        // [kRT][D]
  float* s_u = s_q + kRT * D;                         // [kRT][D]
  float* s_p = s_u + kRT * D;                         // [kRT][kBT]
  float* s_m = s_p + kRT * kBT;
  float* s_z = s_m + kRT;
  float* s_a = s_z + kRT;
  int* s_pre = reinterpret_cast<int*>(s_a + kRT);     // [B + 1]

  if (threadIdx.x < 32) warp_block_prefix(p.lengths, p.B, p.N_cap, kBT, s_pre);
  __syncthreads();

  const int H = p.H;
  const CtaRange cr = cta_range(s_pre, p.B, H, p.ctas, blockIdx.x);
  if (cr.g0 >= cr.g1) return;
  const int rt = blockIdx.y;
  const int r0 = rt * kRT;
  const int rows = min(kRT, p.R - r0);
  const int qmax = p.bits == 4 ? 7 : 127;
  const int ngv = p.Dp / p.group;

  int b = find_seq(s_pre, p.B, H, cr.g0);
  int nb = s_pre[b + 1] - s_pre[b];
  const long long off = cr.g0 - static_cast<long long>(H) * s_pre[b];
  int h = static_cast<int>(off / nb);
  int j = static_cast<int>(off % nb);
  long long g = cr.g0;

  while (g < cr.g1) {
    const int len = clamp_len(p.lengths[b], p.N_cap);
    const int j_begin = j;
    const int j_end = static_cast<int>(min(static_cast<long long>(nb), j + (cr.g1 - g)));
    const bool whole = (j_begin == 0) && (j_end == nb) && !p.force_partial;
    const long long head = static_cast<long long>(b) * H + h;
    const long long row_base = (static_cast<long long>(b) * H * p.G + static_cast<long long>(h) * p.G) * p.Lq + r0;
    const uint8_t* kc = p.k_codes + head * p.k_codes_head;
    const float* ks = p.k_scales + head * p.k_scales_head;
    const uint8_t* vc = p.v_codes + head * p.v_codes_head;
    const float* vs = p.v_scales + head * p.v_scales_head;

    for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x)
      s_q[idx] = load_as_f32(p.Q, row_base * D + idx, p.q_dtype);
    for (int idx = threadIdx.x; idx < kRT * D; idx += blockDim.x) s_u[idx] = 0.f;
    if (threadIdx.x < kRT) {
      s_m[threadIdx.x] = -INFINITY;
      s_z[threadIdx.x] = 0.f;
    }
    __syncthreads();

    for (; j < j_end; ++j) {
      const int t_base = j * kBT;
      const int nt = min(kBT, len - t_base);
      // decode the block's K and V into shared memory, kU elements a thread
      // per round with every load of the round issued before any use
      constexpr int kU = 4;
      for (int i0 = 0; i0 < kBT * D; i0 += kU * kThreads) {
        int kcode[kU], vcode[kU];
        float ksc[kU], vsc[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int idx = i0 + u * kThreads + static_cast<int>(threadIdx.x);
          const int t = idx / D, d = idx - t * D;
          kcode[u] = vcode[u] = 0;
          ksc[u] = vsc[u] = 0.f;
          if (idx < kBT * D && t < nt) {
            const long long tok = t_base + t;
            kcode[u] = code_at(kc, tok * D + d, p.bits);
            ksc[u] = ks[(tok / p.group) * D + d];
            vcode[u] = code_at(vc, tok * p.Dp + d, p.bits);
            vsc[u] = vs[tok * ngv + d / p.group];
          }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int idx = i0 + u * kThreads + static_cast<int>(threadIdx.x);
          if (idx < kBT * D) {
            const int t = idx / D, d = idx - t * D;
            const bool in = t < nt;
            s_k[t * DS + d] = in ? __fmul_rn(static_cast<float>(kcode[u]) - static_cast<float>(qmax), ksc[u]) : 0.f;
            s_v[t * DS + d] = in ? __fmul_rn(static_cast<float>(vcode[u]) - static_cast<float>(qmax), vsc[u]) : 0.f;
          }
        }
      }
      __syncthreads();
      for (int idx = threadIdx.x; idx < kRT * kBT; idx += blockDim.x) {
        const int r = idx / kBT, t = idx - r * kBT;
        float sc = -INFINITY;
        // causal: key t_base + t is visible to query (r0 + r) % Lq up to its position
        const bool seen = !p.causal || t_base + t <= len - p.Lq + (r0 + r) % p.Lq;
        if (r < rows && t < nt && seen) {
          float acc = 0.f;
          for (int d = 0; d < D; ++d) acc = fmaf(s_q[r * D + d], s_k[t * DS + d], acc);
          sc = acc * p.scale;
        }
        s_p[idx] = sc;
      }
      __syncthreads();
      // the block rule per row: a warp per row, lane t = token t (kBT = 32)
      static_assert(kBT == 32, "one token per lane");
      for (int r = static_cast<int>(threadIdx.x >> 5); r < rows; r += kThreads / 32) {
        const int t = static_cast<int>(threadIdx.x & 31);
        const float sc = t < nt ? s_p[r * kBT + t] : -INFINITY;
        float mb = sc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
        const float mo = s_m[r];
        const float mn = fmaxf(mo, mb);
        // a masked key is -inf, and so is mn while a causal row has seen no key
        const float e = sc != -INFINITY ? expf(sc - mn) : 0.f;
        s_p[r * kBT + t] = e;
        float zs = e;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
        __syncwarp();
        if (t == 0) {
          const float a = (mo == -INFINITY) ? 0.f : expf(mo - mn);
          s_z[r] = a * s_z[r] + zs;
          s_m[r] = mn;
          s_a[r] = a;
        }
      }
      __syncthreads();
      for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x) {
        const int r = idx / D, d = idx - r * D;
        float acc = s_a[r] * s_u[idx];
        for (int t = 0; t < nt; ++t) acc = fmaf(s_p[r * kBT + t], s_v[t * DS + d], acc);
        s_u[idx] = acc;
      }
      __syncthreads();
    }

    if (whole) {
      for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x) {
        const int r = idx / D;
        // z = 0: a causal row with no visible key (length < Lq, reported by the merge)
        store_from_f32(p.O, row_base * D + idx, s_z[r] > 0.f ? s_u[idx] / s_z[r] : 0.f, p.q_dtype);
      }
    } else {
      const long long slot = static_cast<long long>(blockIdx.x) + head;
      float* part = p.partials + (slot * p.n_rt + rt) * kRT * (D + 2);
      for (int idx = threadIdx.x; idx < rows * (D + 2); idx += blockDim.x) {
        const int r = idx / (D + 2), e = idx - r * (D + 2);
        part[idx] = e == 0 ? s_m[r] : (e == 1 ? s_z[r] : s_u[r * D + e - 2]);
      }
    }
    __syncthreads();

    g += j_end - j_begin;
    if (j_end == nb) {
      j = 0;
      if (++h == H) {
        h = 0;
        ++b;
        while (b < p.B && s_pre[b + 1] == s_pre[b]) ++b;
        if (b >= p.B) break;
        nb = s_pre[b + 1] - s_pre[b];
      }
    }
  }
}

int rows_per_head(const AttendArgs& a) { return (a.H_q / a.g.H_kv) * a.Lq; }

int generic_ctas(const AttendArgs& a) {
  const int R = rows_per_head(a);
  const int n_rt = (R + kRT - 1) / kRT;
  const long long t_max = static_cast<long long>(a.g.B) * a.g.H_kv * ((a.g.N_cap + kBT - 1) / kBT);
  long long ctas = a.splits > 0 ? a.splits : (2LL * (sm_count() > 0 ? sm_count() : 148) + n_rt - 1) / n_rt;
  if (ctas > t_max) ctas = t_max;
  if (ctas < 1) ctas = 1;
  return static_cast<int>(ctas);
}

bool generic_applies(const AttendArgs& a) { return a.g.D <= 256; }

size_t generic_workspace(const AttendArgs& a) {
  const int R = rows_per_head(a);
  const int n_rt = (R + kRT - 1) / kRT;
  return with_window_slots(a, partial_slots(generic_ctas(a), a.g.B, a.g.H_kv),
                           static_cast<size_t>(n_rt) * kRT * (a.g.D + 2) * sizeof(float));
}

kvq_status generic_launch(const AttendArgs& a, cudaStream_t s) {
  const int R = rows_per_head(a);
  const int n_rt = (R + kRT - 1) / kRT;
  const int ctas = generic_ctas(a);
  const size_t smem = smem_bytes(a.g.D, a.g.B);
  if (smem > 227 * 1024) return KVQ_ERR_UNSUPPORTED;
  if (n_rt > 65535) return KVQ_ERR_UNSUPPORTED;
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(attend_generic_kernel), smem)) return KVQ_ERR_CUDA;
  GenericParams p{};
  p.Q = a.Q;
  p.q_dtype = a.q_dtype;
  p.k_codes = a.k_codes;
  p.k_scales = a.k_scales;
  p.v_codes = a.v_codes;
  p.v_scales = a.v_scales;
  p.lengths = a.lengths;
  p.bits = a.g.bits;
  p.group = a.g.group;
  p.B = a.g.B;
  p.H = a.g.H_kv;
  p.N_cap = a.g.N_cap;
  p.D = a.g.D;
  p.Dp = a.g.Dp;
  p.k_codes_head = static_cast<long long>(a.g.k_codes_head);
  p.k_scales_head = static_cast<long long>(a.g.k_scales_head);
  p.v_codes_head = static_cast<long long>(a.g.v_codes_head);
  p.v_scales_head = static_cast<long long>(a.g.v_scales_head);
  p.G = a.H_q / a.g.H_kv;
  p.Lq = a.Lq;
  p.R = R;
  p.n_rt = n_rt;
  p.scale = a.scale;
  p.O = a.O;
  p.partials = static_cast<float*>(a.workspace);
  p.ctas = ctas;
  p.force_partial = a.win_lengths != nullptr;
  p.causal = a.causal;
  const cudaError_t le = launch_pdl(attend_generic_kernel, dim3(ctas, n_rt), dim3(kThreads), smem, s, p);
  if (le != cudaSuccess) return KVQ_ERR_CUDA;
  count_launch();

  MergeArgs m{};
  m.partials = static_cast<const float*>(a.workspace);
  m.lengths = a.lengths;
  m.O = a.O;
  m.o_dtype = a.q_dtype;
  m.B = a.g.B;
  m.H_kv = a.g.H_kv;
  m.N_cap = a.g.N_cap;
  m.BT = kBT;
  m.ctas = ctas;
  m.R = R;
  m.R_pad = n_rt * kRT;
  m.D = a.g.D;
  m.G = p.G;
  m.Lq = a.Lq;
  m.causal = a.causal;
  const kvq_status ws = add_window(a, p.partials, static_cast<long long>(partial_slots(ctas, a.g.B, a.g.H_kv)),
                                   static_cast<long long>(n_rt) * kRT * (a.g.D + 2), a.g.D + 2,
                                   32LL * (a.g.D + 2), 1, &m, s);
  if (ws != KVQ_OK) return ws;
  return launch_merge(m, s);
}

const AttendImpl kGeneric{"generic", generic_applies, generic_workspace, generic_launch};

}  // namespace

const AttendImpl& generic_attend_impl() { return kGeneric; }

}  // namespace kvq

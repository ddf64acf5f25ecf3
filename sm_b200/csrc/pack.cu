// Quantize-and-pack kernels ("KV分组打包：4-bit到底省了多少？",
// huhohoo.com/docs/llm/kv-packed-groups, sections "一个字节里到底装了什么" and
// "为什么分组要同时看方向与长度").
//
// scale = max|x| / qmax per group in IEEE float32 (1 for an all-zero group),
// code = clip(rint(x / scale), -qmax, qmax) + qmax with a correctly rounded
// division and ties-to-even rounding, so the bytes match a NumPy float32
// implementation bit for bit.  4-bit codes pair over the flattened padded
// code matrix of each (b, h): byte j = code[2j] | code[2j+1] << 4.
#include "kvq_internal.cuh"
#include "quant.cuh"

namespace kvq {
namespace {

struct PackParams {
  const void* X;
  int dtype;
  int t0, T;                 // first token, tokens in the input
  int bits, group, B, H, D, Dp;
  long long codes_head, scales_head;
  uint8_t* codes;
  float* scales;
};

// K: one CTA per (group of g tokens, h, b).  Scales run along tokens within
// each channel; the group's codes are g*D consecutive entries of the
// flattened Np x D code matrix, so a 4-bit group owns whole bytes (g even).
__global__ void __launch_bounds__(256) pack_k_kernel(PackParams p) {
  griddep_wait();
  extern __shared__ float s_x[];                   // [g][D], then scale[D], 1/scale[D]
  const int gi = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = p.group, D = p.D;
  const int qmax = p.bits == 4 ? 7 : 127;
  const long long head = static_cast<long long>(b) * p.H + h;
  const long long in_base = head * p.T * D;
  const int tt0 = gi * g;
  // the group's g x D inputs into shared memory, loads issued in batches so
  // their latencies overlap (float4 when the input is f32, 16-byte aligned
  // and the group lies inside the range)
  const int n = g * D;
  const float* xf = static_cast<const float*>(p.X) + in_base + static_cast<long long>(tt0) * D;
  if (p.dtype == KVQ_F32 && (D & 3) == 0 && tt0 + g <= p.T && (reinterpret_cast<uintptr_t>(xf) & 15u) == 0) {
    const float4* src = reinterpret_cast<const float4*>(xf);
    float4* dst = reinterpret_cast<float4*>(s_x);
    constexpr int U = 4;
    for (int i0 = 0; i0 < n / 4; i0 += U * static_cast<int>(blockDim.x)) {
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * static_cast<int>(blockDim.x) + threadIdx.x;
        v[u] = i < n / 4 ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * static_cast<int>(blockDim.x) + threadIdx.x;
        if (i < n / 4) dst[i] = v[u];
      }
    }
  } else {
    constexpr int U = 8;
    for (int i0 = 0; i0 < n; i0 += U * static_cast<int>(blockDim.x)) {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int idx = i0 + u * static_cast<int>(blockDim.x) + threadIdx.x;
        const int tt = tt0 + idx / D;
        v[u] = (idx < n && tt < p.T) ? load_as_f32(p.X, in_base + static_cast<long long>(tt) * D + idx % D, p.dtype)
                                     : 0.f;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int idx = i0 + u * static_cast<int>(blockDim.x) + threadIdx.x;
        if (idx < n) s_x[idx] = v[u];
      }
    }
  }
  __syncthreads();
  float* s_scale = s_x + g * D;
  const long long kgroup = p.t0 / g + gi;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float amax = 0.f;
#pragma unroll 8
    for (int tt = 0; tt < g; ++tt) amax = fmaxf(amax, fabsf(s_x[tt * D + d]));
    const float sc = group_scale(amax, qmax);
    s_scale[d] = sc;
    s_scale[D + d] = __frcp_rn(sc);
    p.scales[head * p.scales_head + kgroup * D + d] = sc;
  }
  __syncthreads();
  const long long code0 = (static_cast<long long>(p.t0) + tt0) * D;   // flat index of the group start
  uint8_t* out = p.codes + head * p.codes_head;
  if (p.bits == 4) {
    for (int jb = threadIdx.x; jb < g * D / 2; jb += blockDim.x) {
      const int f = 2 * jb;
      const int d0 = f % D, d1 = (f + 1) % D;
      const unsigned lo = quant_code(s_x[f], s_scale[d0], s_scale[D + d0], qmax);
      const unsigned hi = quant_code(s_x[f + 1], s_scale[d1], s_scale[D + d1], qmax);
      out[code0 / 2 + jb] = static_cast<uint8_t>(lo | (hi << 4));
    }
  } else {
    for (int f = threadIdx.x; f < g * D; f += blockDim.x)
      out[code0 + f] = static_cast<uint8_t>(quant_code(s_x[f], s_scale[f % D], s_scale[D + f % D], qmax));
  }
}

// V: one thread per (token, group of g features).  Features beyond D are the
// zero padding of the last group.
__global__ void __launch_bounds__(256) pack_v_kernel(PackParams p) {
  griddep_wait();
  const int ng = p.Dp / p.group;
  const long long total = static_cast<long long>(p.B) * p.H * p.T * ng;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int g = p.group, D = p.D;
  const int qmax = p.bits == 4 ? 7 : 127;
  const int gj = static_cast<int>(idx % ng);
  const long long row = idx / ng;                 // (b*H + h)*T + tt
  const long long head = row / p.T;
  const int tt = static_cast<int>(row % p.T);
  const long long in_base = row * D;
  const int d0 = gj * g;
  float amax = 0.f;
  for (int e = 0; e < g; ++e) {
    const int d = d0 + e;
    if (d < D) amax = fmaxf(amax, fabsf(load_as_f32(p.X, in_base + d, p.dtype)));
  }
  const float sc = group_scale(amax, qmax);
  const float rs = __frcp_rn(sc);
  const long long tok = static_cast<long long>(p.t0) + tt;
  p.scales[head * p.scales_head + tok * ng + gj] = sc;
  const long long code0 = tok * p.Dp + d0;
  uint8_t* out = p.codes + head * p.codes_head;
  if (p.bits == 4) {
    for (int e = 0; e < g; e += 2) {
      const float x0 = d0 + e < D ? load_as_f32(p.X, in_base + d0 + e, p.dtype) : 0.f;
      const float x1 = d0 + e + 1 < D ? load_as_f32(p.X, in_base + d0 + e + 1, p.dtype) : 0.f;
      out[(code0 + e) / 2] =
          static_cast<uint8_t>(quant_code(x0, sc, rs, qmax) | (quant_code(x1, sc, rs, qmax) << 4));
    }
  } else {
    for (int e = 0; e < g; ++e) {
      const float x = d0 + e < D ? load_as_f32(p.X, in_base + d0 + e, p.dtype) : 0.f;
      out[code0 + e] = static_cast<uint8_t>(quant_code(x, sc, rs, qmax));
    }
  }
}

// V, D = 128 and groups of 32: one warp per token row.  Lane l holds features
// 4l..4l+3 (one 16-byte load), the 8 lanes of a group reduce the group max
// with shuffles, and the lane writes its 4 codes (2 bytes, or 4 at 8 bits).
__global__ void __launch_bounds__(256) pack_v128_kernel(PackParams p) {
  griddep_wait();
  const long long rows = static_cast<long long>(p.B) * p.H * p.T;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int qmax = p.bits == 4 ? 7 : 127;
  float x[4];
  if (p.dtype == KVQ_F32) {
    const float4 v = reinterpret_cast<const float4*>(p.X)[row * 32 + lane];
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else {
    const uint2 v = reinterpret_cast<const uint2*>(p.X)[row * 32 + lane];
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xFFFF0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  }
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
  const float sc = group_scale(amax, qmax);
  const float rs = __frcp_rn(sc);
  const long long head = row / p.T;
  const long long tok = static_cast<long long>(p.t0) + row % p.T;
  if ((lane & 7) == 0) p.scales[head * p.scales_head + tok * 4 + (lane >> 3)] = sc;
  unsigned c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = quant_code(x[i], sc, rs, qmax);
  uint8_t* out = p.codes + head * p.codes_head;
  if (p.bits == 4) {
    reinterpret_cast<uint16_t*>(out + tok * 64)[lane] =
        static_cast<uint16_t>(c[0] | (c[1] << 4) | (c[2] << 8) | (c[3] << 12));
  } else {
    reinterpret_cast<uint32_t*>(out + tok * 128)[lane] = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
  }
}

// Decode-step append: one CTA per (h, b).  Sequence b's new token sits at
// t = lengths[b] - 1.  The CTA re-packs K group t / g from the caller's
// float rows of that group (rows past t % g read as zero, as a whole-cache
// pack pads a short last group) and packs V row t; what it writes is exactly
// what kvq_pack of tokens [0, lengths[b]) writes for that group and row.
struct AppendParams {
  const void* K_tail;        // [B, H, g, D]
  const void* V_new;         // [B, H, D]
  int dtype;
  const int32_t* lengths;
  int bits, group, B, H, D, Dp, N_cap;
  long long k_codes_head, k_scales_head, v_codes_head, v_scales_head;
  uint8_t* k_codes;
  float* k_scales;
  uint8_t* v_codes;
  float* v_scales;
  unsigned int* err;
};

__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
  griddep_wait();
  extern __shared__ float s_x[];                   // [g][D] tail rows, then scale[D], 1/scale[D]
  const int h = blockIdx.x, b = blockIdx.y;
  const int L = p.lengths[b];
  if (L < 1 || L > p.N_cap) {
    if (threadIdx.x == 0 && h == 0) record_error(p.err, KVQ_ERR_LENGTH);
    return;
  }
  const int g = p.group, D = p.D;
  const int qmax = p.bits == 4 ? 7 : 127;
  const int t = L - 1, j = t / g, nin = t % g + 1;
  const long long head = static_cast<long long>(b) * p.H + h;

  // K: the group's rows into shared memory, loads issued in batches
  const int n = g * D;
  const long long kin = head * n;
  constexpr int U = 8;
  for (int i0 = 0; i0 < n; i0 += U * static_cast<int>(blockDim.x)) {
    float v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * static_cast<int>(blockDim.x) + threadIdx.x;
      v[u] = (i < n && i / D < nin) ? load_as_f32(p.K_tail, kin + i, p.dtype) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * static_cast<int>(blockDim.x) + threadIdx.x;
      if (i < n) s_x[i] = v[u];
    }
  }
  __syncthreads();
  float* s_scale = s_x + n;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float amax = 0.f;
    for (int tt = 0; tt < nin; ++tt) amax = fmaxf(amax, fabsf(s_x[tt * D + d]));
    const float sc = group_scale(amax, qmax);
    s_scale[d] = sc;
    s_scale[D + d] = __frcp_rn(sc);
    p.k_scales[head * p.k_scales_head + static_cast<long long>(j) * D + d] = sc;
  }
  __syncthreads();
  const long long code0 = static_cast<long long>(j) * n;           // flat index of the group start
  uint8_t* kout = p.k_codes + head * p.k_codes_head;
  if (p.bits == 4) {
    for (int jb = threadIdx.x; jb < n / 2; jb += blockDim.x) {
      const int f = 2 * jb;
      const int d0 = f % D, d1 = (f + 1) % D;
      const unsigned lo = quant_code(s_x[f], s_scale[d0], s_scale[D + d0], qmax);
      const unsigned hi = quant_code(s_x[f + 1], s_scale[d1], s_scale[D + d1], qmax);
      kout[code0 / 2 + jb] = static_cast<uint8_t>(lo | (hi << 4));
    }
  } else {
    for (int f = threadIdx.x; f < n; f += blockDim.x)
      kout[code0 + f] = static_cast<uint8_t>(quant_code(s_x[f], s_scale[f % D], s_scale[D + f % D], qmax));
  }

  // V row t: warp w takes feature groups w, w + warps, ...; features past D
  // are the zero padding of the last group
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int ng = p.Dp / g;
  const long long vin = head * D;
  uint8_t* vout = p.v_codes + head * p.v_codes_head;
  for (int gj = warp; gj < ng; gj += nw) {
    const int d0 = gj * g;
    float amax = 0.f;
    for (int e = lane; e < g; e += 32)
      if (d0 + e < D) amax = fmaxf(amax, fabsf(load_as_f32(p.V_new, vin + d0 + e, p.dtype)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = group_scale(amax, qmax);
    const float rs = __frcp_rn(sc);
    if (lane == 0) p.v_scales[head * p.v_scales_head + static_cast<long long>(t) * ng + gj] = sc;
    const long long c0 = static_cast<long long>(t) * p.Dp + d0;     // even: Dp and d0 are multiples of g
    if (p.bits == 4) {
      for (int e = 2 * lane; e < g; e += 64) {
        const float x0 = d0 + e < D ? load_as_f32(p.V_new, vin + d0 + e, p.dtype) : 0.f;
        const float x1 = d0 + e + 1 < D ? load_as_f32(p.V_new, vin + d0 + e + 1, p.dtype) : 0.f;
        vout[(c0 + e) / 2] = static_cast<uint8_t>(quant_code(x0, sc, rs, qmax) | (quant_code(x1, sc, rs, qmax) << 4));
      }
    } else {
      for (int e = lane; e < g; e += 32) {
        const float x = d0 + e < D ? load_as_f32(p.V_new, vin + d0 + e, p.dtype) : 0.f;
        vout[c0 + e] = static_cast<uint8_t>(quant_code(x, sc, rs, qmax));
      }
    }
  }
}

}  // namespace

size_t append_smem_bytes(const Geometry& g) {
  return (static_cast<size_t>(g.group) * g.D + 2 * static_cast<size_t>(g.D)) * sizeof(float);
}

kvq_status launch_append(const AppendArgs& a, cudaStream_t s) {
  const Geometry& g = a.g;
  if (g.B > 65535 || g.H_kv > 65535) return KVQ_ERR_UNSUPPORTED;
  const size_t smem = append_smem_bytes(g);
  if (smem > 227 * 1024) return KVQ_ERR_UNSUPPORTED;
  if (smem > 48 * 1024 && !ensure_dynamic_smem(reinterpret_cast<const void*>(append_kernel), smem))
    return KVQ_ERR_CUDA;
  AppendParams p{};
  p.K_tail = a.K_tail;
  p.V_new = a.V_new;
  p.dtype = a.in_dtype;
  p.lengths = a.lengths;
  p.bits = g.bits;
  p.group = g.group;
  p.B = g.B;
  p.H = g.H_kv;
  p.D = g.D;
  p.Dp = g.Dp;
  p.N_cap = g.N_cap;
  p.k_codes_head = static_cast<long long>(g.k_codes_head);
  p.k_scales_head = static_cast<long long>(g.k_scales_head);
  p.v_codes_head = static_cast<long long>(g.v_codes_head);
  p.v_scales_head = static_cast<long long>(g.v_scales_head);
  p.k_codes = a.k_codes;
  p.k_scales = a.k_scales;
  p.v_codes = a.v_codes;
  p.v_scales = a.v_scales;
  p.err = error_word();
  if (!p.err) return KVQ_ERR_CUDA;
  if (launch_pdl(append_kernel, dim3(g.H_kv, g.B), dim3(256), smem, s, p) != cudaSuccess) return KVQ_ERR_CUDA;
  count_launch();
  return KVQ_OK;
}

kvq_status launch_pack(const PackArgs& a, cudaStream_t s) {
  const Geometry& g = a.g;
  const int T = a.t1 - a.t0;
  if (g.B > 65535 || g.H_kv > 65535) return KVQ_ERR_UNSUPPORTED;
  if (a.K) {
    const size_t smem = (static_cast<size_t>(g.group) * g.D + 2 * g.D) * sizeof(float);
    if (smem > 227 * 1024) return KVQ_ERR_UNSUPPORTED;
    if (smem > 48 * 1024) {
      if (!ensure_dynamic_smem(reinterpret_cast<const void*>(pack_k_kernel), smem)) return KVQ_ERR_CUDA;
    }
    PackParams pk{a.K, a.in_dtype, a.t0, T, g.bits, g.group, g.B, g.H_kv, g.D, g.Dp,
                  static_cast<long long>(g.k_codes_head), static_cast<long long>(g.k_scales_head),
                  a.k_codes, a.k_scales};
    const dim3 kgrid((T + g.group - 1) / g.group, g.H_kv, g.B);
    if (launch_pdl(pack_k_kernel, kgrid, dim3(256), smem, s, pk) != cudaSuccess) return KVQ_ERR_CUDA;
    count_launch();
  }
  if (a.V) {
    PackParams pv{a.V, a.in_dtype, a.t0, T, g.bits, g.group, g.B, g.H_kv, g.D, g.Dp,
                  static_cast<long long>(g.v_codes_head), static_cast<long long>(g.v_scales_head),
                  a.v_codes, a.v_scales};
    const size_t esz = a.in_dtype == KVQ_F32 ? 4 : 2;
    const bool fast = g.D == 128 && g.group == 32 &&
                      (reinterpret_cast<uintptr_t>(a.V) % (4 * esz)) == 0 &&
                      (reinterpret_cast<uintptr_t>(a.v_codes) % 4) == 0;
    if (fast) {
      const long long rows = static_cast<long long>(g.B) * g.H_kv * T;
      const long long blocks = (rows + 7) / 8;
      if (blocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
      if (launch_pdl(pack_v128_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, pv) != cudaSuccess)
        return KVQ_ERR_CUDA;
    } else {
      const long long vthreads = static_cast<long long>(g.B) * g.H_kv * T * (g.Dp / g.group);
      const long long vblocks = (vthreads + 255) / 256;
      if (vblocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
      if (launch_pdl(pack_v_kernel, dim3(static_cast<unsigned>(vblocks)), dim3(256), 0, s, pv) != cudaSuccess)
        return KVQ_ERR_CUDA;
    }
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
  }
  return KVQ_OK;
}

}  // namespace kvq

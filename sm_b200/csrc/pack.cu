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

namespace kvq {
namespace {

__device__ __forceinline__ unsigned quant_code(float x, float s, int qmax) {
  float q = rintf(__fdiv_rn(x, s));
  q = fminf(fmaxf(q, -static_cast<float>(qmax)), static_cast<float>(qmax));
  return static_cast<unsigned>(static_cast<int>(q) + qmax);
}

__device__ __forceinline__ float group_scale(float amax, int qmax) {
  return amax == 0.f ? 1.f : __fdiv_rn(amax, static_cast<float>(qmax));
}

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
  extern __shared__ float s_x[];                   // [g][D] then scale[D]
  const int gi = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = p.group, D = p.D;
  const int qmax = p.bits == 4 ? 7 : 127;
  const long long head = static_cast<long long>(b) * p.H + h;
  const long long in_base = head * p.T * D;
  const int tt0 = gi * g;
  for (int idx = threadIdx.x; idx < g * D; idx += blockDim.x) {
    const int tt = tt0 + idx / D;
    const int d = idx % D;
    s_x[idx] = tt < p.T ? load_as_f32(p.X, in_base + static_cast<long long>(tt) * D + d, p.dtype) : 0.f;
  }
  __syncthreads();
  float* s_scale = s_x + g * D;
  const long long kgroup = p.t0 / g + gi;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float amax = 0.f;
    for (int tt = 0; tt < g; ++tt) amax = fmaxf(amax, fabsf(s_x[tt * D + d]));
    const float sc = group_scale(amax, qmax);
    s_scale[d] = sc;
    p.scales[head * p.scales_head + kgroup * D + d] = sc;
  }
  __syncthreads();
  const long long code0 = (static_cast<long long>(p.t0) + tt0) * D;   // flat index of the group start
  uint8_t* out = p.codes + head * p.codes_head;
  if (p.bits == 4) {
    for (int jb = threadIdx.x; jb < g * D / 2; jb += blockDim.x) {
      const int f = 2 * jb;
      const unsigned lo = quant_code(s_x[f], s_scale[f % D], qmax);
      const unsigned hi = quant_code(s_x[f + 1], s_scale[(f + 1) % D], qmax);
      out[code0 / 2 + jb] = static_cast<uint8_t>(lo | (hi << 4));
    }
  } else {
    for (int f = threadIdx.x; f < g * D; f += blockDim.x)
      out[code0 + f] = static_cast<uint8_t>(quant_code(s_x[f], s_scale[f % D], qmax));
  }
}

// V: one thread per (token, group of g features).  Features beyond D are the
// zero padding of the last group.
__global__ void __launch_bounds__(256) pack_v_kernel(PackParams p) {
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
  const long long tok = static_cast<long long>(p.t0) + tt;
  p.scales[head * p.scales_head + tok * ng + gj] = sc;
  const long long code0 = tok * p.Dp + d0;
  uint8_t* out = p.codes + head * p.codes_head;
  if (p.bits == 4) {
    for (int e = 0; e < g; e += 2) {
      const float x0 = d0 + e < D ? load_as_f32(p.X, in_base + d0 + e, p.dtype) : 0.f;
      const float x1 = d0 + e + 1 < D ? load_as_f32(p.X, in_base + d0 + e + 1, p.dtype) : 0.f;
      out[(code0 + e) / 2] = static_cast<uint8_t>(quant_code(x0, sc, qmax) | (quant_code(x1, sc, qmax) << 4));
    }
  } else {
    for (int e = 0; e < g; ++e) {
      const float x = d0 + e < D ? load_as_f32(p.X, in_base + d0 + e, p.dtype) : 0.f;
      out[code0 + e] = static_cast<uint8_t>(quant_code(x, sc, qmax));
    }
  }
}

}  // namespace

kvq_status launch_pack(const PackArgs& a, cudaStream_t s) {
  const Geometry& g = a.g;
  const int T = a.t1 - a.t0;
  const size_t smem = (static_cast<size_t>(g.group) * g.D + g.D) * sizeof(float);
  if (smem > 227 * 1024) return KVQ_ERR_UNSUPPORTED;
  if (g.B > 65535 || g.H_kv > 65535) return KVQ_ERR_UNSUPPORTED;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(pack_k_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return KVQ_ERR_CUDA;
  }
  PackParams pk{a.K, a.in_dtype, a.t0, T, g.bits, g.group, g.B, g.H_kv, g.D, g.Dp,
                static_cast<long long>(g.k_codes_head), static_cast<long long>(g.k_scales_head),
                a.k_codes, a.k_scales};
  const dim3 kgrid((T + g.group - 1) / g.group, g.H_kv, g.B);
  pack_k_kernel<<<kgrid, 256, smem, s>>>(pk);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;

  PackParams pv{a.V, a.in_dtype, a.t0, T, g.bits, g.group, g.B, g.H_kv, g.D, g.Dp,
                static_cast<long long>(g.v_codes_head), static_cast<long long>(g.v_scales_head),
                a.v_codes, a.v_scales};
  const long long vthreads = static_cast<long long>(g.B) * g.H_kv * T * (g.Dp / g.group);
  const long long vblocks = (vthreads + 255) / 256;
  if (vblocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  pack_v_kernel<<<static_cast<unsigned>(vblocks), 256, 0, s>>>(pv);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
  return KVQ_OK;
}

}  // namespace kvq

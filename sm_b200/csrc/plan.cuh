// Work plan over the concatenated (b, h, token-block) list, device side.
//
// Blocks of BT tokens are listed sequence-major, then KV head, then block
// index.  With pre[b] = number of blocks of sequences 0..b-1, the blocks of
// (b, h) are the global indices [H*pre[b] + h*nb, H*pre[b] + (h+1)*nb),
// nb = pre[b+1] - pre[b].  CTA c of `ctas` owns [c*P, min((c+1)*P, T)) with
// T = H*pre[B] and P = ceil(T / ctas), so every CTA gets the same number of
// blocks (up to one) whatever the lengths.  A (b, h) covered by several CTAs
// is finished by merging their partial (m, z, u) states with the block rule.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// Warp 0 fills pre[0..B] (the caller synchronises the CTA afterwards).
// l2: read the lengths at the L2 (ld.global.cg), as a kernel does that reads
// them before its grid-dependency wait.  extra: slots added per head of every
// sequence with a length in [1, n_cap] -- the decode step's append, counted
// as work in the split so the workers that append cover fewer blocks (no
// block sits in such a slot: a worker's blocks of a head stop at the head's
// last real block).
__device__ __forceinline__ void warp_block_prefix(const int32_t* lengths, int B, int n_cap, int bt,
                                                  int* pre, bool l2 = false, int extra = 0) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 0; base < B; base += 32) {
    const int b = base + lane;
    int v = 0;
    if (b < B) {
      const int raw = l2 ? __ldcg(lengths + b) : __ldg(lengths + b);
      v = seq_blocks(raw, n_cap, bt) + ((raw >= 1 && raw <= n_cap) ? extra : 0);
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (b < B) pre[b + 1] = carry + v;
    carry += __shfl_sync(0xffffffffu, v, 31);
  }
  if (lane == 0) pre[0] = 0;
}

// Largest b in [0, B) with H*pre[b] <= gidx.
__device__ __forceinline__ int find_seq(const int* pre, int B, int H, long long gidx) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<long long>(H) * pre[mid] <= gidx) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

struct CtaRange {
  long long g0, g1, P, T;
};

__device__ __forceinline__ CtaRange cta_range(const int* pre, int B, int H, int ctas, int c) {
  CtaRange r;
  r.T = static_cast<long long>(H) * pre[B];
  r.P = (r.T + ctas - 1) / ctas;
  r.g0 = static_cast<long long>(c) * r.P;
  r.g1 = r.T < r.g0 + r.P ? r.T : r.g0 + r.P;
  return r;
}

__device__ __forceinline__ int clamp_len(int len, int n_cap) {
  return len < 0 ? 0 : (len > n_cap ? n_cap : len);
}

}  // namespace kvq

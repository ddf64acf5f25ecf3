// Group quantization arithmetic shared by every kernel that writes the packed
// cache ("KV分组打包：4-bit到底省了多少？", huhohoo.com/docs/llm/kv-packed-groups,
// section "一个字节里到底装了什么"): scale = max|x| / qmax in IEEE float32 (1
// for an all-zero group) and code = clip(rint(x / scale), -qmax, qmax) + qmax
// with a correctly rounded quotient, so the bytes match a NumPy float32
// implementation bit for bit whichever kernel writes them.
#pragma once

namespace kvq {

// rint(x / s) with x / s correctly rounded first.  x * (1/s) is within a few
// ulps of x / s, and |x / s| <= 127, so its error stays below 2^-15: unless it
// lies within 2^-12 of a rounding tie it rounds to the same integer as the
// correctly rounded quotient.  Near a tie (or if 1/s overflowed) the exact
// IEEE division decides.
__device__ __forceinline__ unsigned quant_code(float x, float s, float rs, int qmax) {
  const float qa = x * rs;
  float q = rintf(qa);
  const float d = fabsf(qa - q);
  if (!(d < 0.5f - 0.000244140625f)) q = rintf(__fdiv_rn(x, s));
  q = fminf(fmaxf(q, -static_cast<float>(qmax)), static_cast<float>(qmax));
  return static_cast<unsigned>(static_cast<int>(q) + qmax);
}

__device__ __forceinline__ float group_scale(float amax, int qmax) {
  return amax == 0.f ? 1.f : __fdiv_rn(amax, static_cast<float>(qmax));
}

}  // namespace kvq

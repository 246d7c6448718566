// Device pieces of the ES-dLLM selection shared by the standalone kernels and the
// fused layer-run kernel, so both score and rank a row with the same arithmetic.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace dllm {

// Monotone map of a score to uint32 (larger score -> larger key): NaN lowest, -0 == +0.
__device__ __forceinline__ uint32_t order_key(float x) {
  if (x != x) return 0u;
  x = x + 0.0f;
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float es_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Partial sums of ES-dLLM Eq. 1 over columns [i0, i1) of one row (i0 a multiple of 128,
// i1 of 4; a warp, each lane 4 columns of every 128): l1 += |x - xp|, l2 += xp^2 (this lane's
// share).  x is the row's input of the scored layer this iteration, xp its input last
// iteration.  update != 0 rolls xp := x.  carried: the previous layer skipped the row, so
// its input is its cached output of that layer, xp itself: x := xp, no l1, xp unchanged.
// Loads bypass L1 (other CTAs of a persistent kernel may have written the rows).
__device__ __forceinline__ void es_eq1_part(float* __restrict__ x, float* __restrict__ xp, int i0, int i1,
                                            int update, bool carried, int lane, float& l1, float& l2) {
  for (int i = i0 + lane * 4; i < i1; i += 128) {
    const float4 b = __ldcg(reinterpret_cast<const float4*>(xp + i));
    l2 += b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
    if (carried) {
      *reinterpret_cast<float4*>(x + i) = b;
      continue;
    }
    const float4 a = __ldcg(reinterpret_cast<const float4*>(x + i));
    l1 += fabsf(a.x - b.x) + fabsf(a.y - b.y) + fabsf(a.z - b.z) + fabsf(a.w - b.w);
    if (update) *reinterpret_cast<float4*>(xp + i) = a;
  }
}

// Eq. 1 from the row's sums:
//   var   = l1 / (sqrt(d) sqrt(l2))   (0 when l2 = 0)
//   score = alpha c + (1 - alpha) var
__device__ __forceinline__ float es_eq1_score(float l1, float l2, int d, float c, float alpha) {
  const float nrm = sqrtf(l2);
  const float var = nrm > 0.f ? l1 / (sqrtf(static_cast<float>(d)) * nrm) : 0.f;
  return alpha * c + (1.f - alpha) * var;
}

// Eq. 1 for one whole row by one warp (every lane gets the score).
__device__ __forceinline__ float es_eq1_row(float* __restrict__ x, float* __restrict__ xp, int d, float c,
                                            float alpha, int update, bool carried, int lane) {
  float l1 = 0.f, l2 = 0.f;
  es_eq1_part(x, xp, 0, d, update, carried, lane, l1, l2);
  return es_eq1_score(es_warp_sum(l1), es_warp_sum(l2), d, c, alpha);
}

}  // namespace dllm

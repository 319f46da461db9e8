// Offline progressive (two-level) weight quantization: fp32 W [N, K] ->
// uint4 codes q, per-group 4-bit zero z and integer scale s2 in [1, 8], and a
// per-output-channel fp16 scale s1, so that W ~ s1 * (q - z) * s2 with
// (q - z) * s2 an exact int8 in [-120, 120] ("QServe/QoQ" abstract:
// progressive quantization keeps W4A8 dequantization cheap).
//
// Level 1 (row n): r_g = max(max W_g, 0) - min(min W_g, 0) per group g of 128;
//   s1 = fp16_rn(max_g r_g / 120); s1 == 0 -> 1; t = W / float(s1).
// Level 2 (group g): lo = min(min t, 0), hi = max(max t, 0);
//   s2 = clamp(ceil((hi - lo) / 15), 1, 8); z = clamp(rint(-lo / s2), 0, 15);
//   q = clamp(rint(t / s2) + z, 0, 15).
// Every divide is an IEEE fp32 divide (round to nearest even).
//
// One CTA per row; one warp per group of 128 (4 floats per lane).
#pragma once
#include "ptx.cuh"

namespace w4a8 {

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int THREADS>
__global__ void __launch_bounds__(THREADS) quantize_weights_kernel(const float* __restrict__ W, int64_t K,
                                                                    uint8_t* __restrict__ q, uint8_t* __restrict__ z,
                                                                    uint8_t* __restrict__ s2,
                                                                    __half* __restrict__ s1) {
  constexpr int WARPS = THREADS / 32;
  __shared__ float red[WARPS];
  const int64_t n = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = static_cast<int>(K >> 7);
  const float4* row = reinterpret_cast<const float4*>(W + n * K);

  // level 1: widest group range of the row
  float rmax = 0.0f;
  for (int g = warp; g < G; g += WARPS) {
    const float4 w = row[g * 32 + lane];
    float lo = fminf(fminf(w.x, w.y), fminf(w.z, w.w));
    float hi = fmaxf(fmaxf(w.x, w.y), fmaxf(w.z, w.w));
    lo = fminf(warp_min(lo), 0.0f);
    hi = fmaxf(warp_max(hi), 0.0f);
    rmax = fmaxf(rmax, __fsub_rn(hi, lo));
  }
  if (lane == 0) red[warp] = rmax;
  __syncthreads();
  float R = 0.0f;
#pragma unroll
  for (int i = 0; i < WARPS; ++i) R = fmaxf(R, red[i]);
  __half s1h = __float2half_rn(__fdiv_rn(R, 120.0f));
  if (__half2float(s1h) == 0.0f) s1h = __float2half_rn(1.0f);
  const float s1f = __half2float(s1h);
  if (threadIdx.x == 0) s1[n] = s1h;

  // level 2, per group
  for (int g = warp; g < G; g += WARPS) {
    const float4 w = row[g * 32 + lane];
    const float t0 = __fdiv_rn(w.x, s1f), t1 = __fdiv_rn(w.y, s1f);
    const float t2 = __fdiv_rn(w.z, s1f), t3 = __fdiv_rn(w.w, s1f);
    const float lo = fminf(warp_min(fminf(fminf(t0, t1), fminf(t2, t3))), 0.0f);
    const float hi = fmaxf(warp_max(fmaxf(fmaxf(t0, t1), fmaxf(t2, t3))), 0.0f);
    const int s2i = max(1, min(8, static_cast<int>(ceilf(__fdiv_rn(__fsub_rn(hi, lo), 15.0f)))));
    const float s2f = static_cast<float>(s2i);
    const int zi = max(0, min(15, __float2int_rn(__fdiv_rn(-lo, s2f))));
    const int q0 = max(0, min(15, __float2int_rn(__fdiv_rn(t0, s2f)) + zi));
    const int q1 = max(0, min(15, __float2int_rn(__fdiv_rn(t1, s2f)) + zi));
    const int q2 = max(0, min(15, __float2int_rn(__fdiv_rn(t2, s2f)) + zi));
    const int q3 = max(0, min(15, __float2int_rn(__fdiv_rn(t3, s2f)) + zi));
    reinterpret_cast<uint32_t*>(q + n * K)[g * 32 + lane] =
        static_cast<uint32_t>(q0) | (static_cast<uint32_t>(q1) << 8) | (static_cast<uint32_t>(q2) << 16) |
        (static_cast<uint32_t>(q3) << 24);
    if (lane == 0) {
      z[n * G + g] = static_cast<uint8_t>(zi);
      s2[n * G + g] = static_cast<uint8_t>(s2i);
    }
  }
}

}  // namespace w4a8

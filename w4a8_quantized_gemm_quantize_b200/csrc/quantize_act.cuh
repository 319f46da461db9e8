// Per-token symmetric int8 quantization of fp16 activations.
//
// Row m: amax = max_k |A|; sA = fp16_rn(amax / 127) (IEEE fp32 divide);
// A8 = clamp(rint(A / float(sA)), -127, 127) (IEEE fp32 divide, rint half to
// even); sA == 0 gives zero codes; rowsum = sum_k A8. This is the dynamic
// per-token 8-bit activation scheme of W4A8 serving ("QServe/QoQ" abstract,
// 8-bit activations; "PrefixQuant ...", Key Findings: per-token dynamic
// quantization).
//
// HBM-bound (2 bytes read + 1 byte written per element). One CTA per row;
// each thread keeps its slice of the row in registers (16-byte vectors), so
// the row is read from HBM once, reduced, then quantized from registers.
#pragma once
#include "ptx.cuh"

namespace w4a8 {

template <int THREADS>
__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < THREADS / 32 ? red[lane] : 0.0f;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  v = red[0];
  __syncthreads();
  return v;
}

template <int THREADS>
__device__ __forceinline__ int block_sum(int v, int* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < THREADS / 32 ? red[lane] : 0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

// Code of one value: clamp(rint(x / sf), -QMAX, QMAX), IEEE fp32 divide,
// ties to even. QMAX = 127 (8-bit codes) or 7 (4-bit codes).
template <int QMAX>
__device__ __forceinline__ int quant_code(float x, float sf) {
  int q = __float2int_rn(__fdiv_rn(x, sf));
  return max(-QMAX, min(QMAX, q));
}

// Codes per token: 8 = one int8 per code (row of K bytes); 4 = two codes per
// byte, code 2j in bits 0-3 and code 2j+1 in bits 4-7 of byte j, 4-bit two's
// complement (row of K / 2 bytes; the W4A4 activations of "PrefixQuant ...",
// Key Findings).
template <int BITS>
struct CodeOut {
  static constexpr int kQmax = BITS == 8 ? 127 : 7;
  // stores the 8 codes of 16-byte input vector idx of a row
  __device__ __forceinline__ static void store(void* row, int idx, const int (&q)[8]) {
    if constexpr (BITS == 8) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j >> 2] |= (static_cast<uint32_t>(q[j]) & 0xFFu) << ((j & 3) * 8);
      reinterpret_cast<uint2*>(row)[idx] = make_uint2(w[0], w[1]);
    } else {
      uint32_t w = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) w |= (static_cast<uint32_t>(q[j]) & 0xFu) << (j * 4);
      reinterpret_cast<uint32_t*>(row)[idx] = w;
    }
  }
};

// VPT: 16-byte vectors (8 halves) per thread; K <= THREADS * VPT * 8.
// BITS: 8 (int8 codes, sA = amax / 127) or 4 (packed 4-bit codes,
// sA = amax / 7).
template <int THREADS, int VPT, int BITS = 8>
__global__ void __launch_bounds__(THREADS) quantize_act_kernel(const __half* __restrict__ A, int64_t K,
                                                                void* __restrict__ codes, __half* __restrict__ sA,
                                                                int32_t* __restrict__ rowsum, int early_release) {
  using Out = CodeOut<BITS>;
  __shared__ float fred[32];
  __shared__ int ird[32];
  // Launched as a programmatic dependent: this grid waits for the preceding
  // kernel's writes before it reads A. With early_release (few tokens, a
  // grid of a few CTAs) the next kernel (the GEMM) may launch right away and
  // stream its weights while this grid runs; it waits for this grid to
  // complete before it reads the codes. A grid of thousands of rows releases
  // it after its wait instead, so that its CTAs do not hold SM slots early.
  if (early_release) grid_launch_dependents();
  grid_dependency_wait();
  if (!early_release) grid_launch_dependents();
  int* ired = ird;
  const int64_t m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(A + m * K);
  const int nvec = static_cast<int>(K >> 3);
  uint4 v[VPT];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * THREADS;
    // streamed once; the address is clamped into the row because the
    // compiler may issue this load ahead of the bounds test
    v[i] = __ldcs(row + (idx < nvec ? idx : nvec - 1));
    if (idx < nvec) {
      const __half2* h = reinterpret_cast<const __half2*>(&v[i]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
  amax = block_max<THREADS>(amax, fred);
  const __half s_h = __float2half_rn(__fdiv_rn(amax, static_cast<float>(Out::kQmax)));
  const float sf = __half2float(s_h);
  int local = 0;
  void* out = static_cast<uint8_t*>(codes) + m * K * BITS / 8;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * THREADS;
    if (idx < nvec) {
      const __half2* h = reinterpret_cast<const __half2*>(&v[i]);
      int q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (sf != 0.0f) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(h[j]);
          q[2 * j] = quant_code<Out::kQmax>(f.x, sf);
          q[2 * j + 1] = quant_code<Out::kQmax>(f.y, sf);
          local += q[2 * j] + q[2 * j + 1];
        }
      }
      Out::store(out, idx, q);
    }
  }
  if (rowsum != nullptr) {
    const int total = block_sum<THREADS>(local, ired);
    if (threadIdx.x == 0) rowsum[m] = total;
  }
  if (threadIdx.x == 0) sA[m] = s_h;
}

// Per-tensor static int8 quantization: one fp16 scale s for the whole tensor,
// fixed offline by calibration ("PrefixQuant: Static Quantization Beats
// Dynamic through Prefixed Outliers in LLMs", Methodology: per-tensor static
// quantization once outlier tokens are prefixed). No amax pass: one read of
// A, A8 = clamp(rint(A / float(s)), -127, 127) (IEEE fp32 divide, ties to
// even; s == 0 gives zero codes), rowsum, and sA[m] = s so that the GEMM's
// per-token epilogue applies the tensor scale. One CTA per token.
template <int THREADS, int VPT, int BITS = 8>
__global__ void __launch_bounds__(THREADS) quantize_act_static_kernel(const __half* __restrict__ A, int64_t K,
                                                                       const __half* __restrict__ s,
                                                                       void* __restrict__ codes,
                                                                       __half* __restrict__ sA,
                                                                       int32_t* __restrict__ rowsum,
                                                                       int early_release) {
  using Out = CodeOut<BITS>;
  __shared__ int ird[32];
  if (early_release) grid_launch_dependents();  // as in quantize_act_kernel
  grid_dependency_wait();                       // A (and s) may come from the preceding kernel
  if (!early_release) grid_launch_dependents();
  const int64_t m = blockIdx.x;
  const __half s_h = *s;
  const float sf = __half2float(s_h);
  const uint4* row = reinterpret_cast<const uint4*>(A + m * K);
  void* out = static_cast<uint8_t*>(codes) + m * K * BITS / 8;
  const int nvec = static_cast<int>(K >> 3);
  int local = 0;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * THREADS;
    // the address is clamped into the row: the load may be issued ahead of
    // the bounds test
    const uint4 v = __ldcs(row + (idx < nvec ? idx : nvec - 1));
    if (idx < nvec) {
      const __half2* h = reinterpret_cast<const __half2*>(&v);
      int q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (sf != 0.0f) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(h[j]);
          q[2 * j] = quant_code<Out::kQmax>(f.x, sf);
          q[2 * j + 1] = quant_code<Out::kQmax>(f.y, sf);
          local += q[2 * j] + q[2 * j + 1];
        }
      }
      Out::store(out, idx, q);
    }
  }
  if (rowsum != nullptr) {
    const int total = block_sum<THREADS>(local, ird);
    if (threadIdx.x == 0) rowsum[m] = total;
  }
  if (threadIdx.x == 0) sA[m] = s_h;
}

}  // namespace w4a8

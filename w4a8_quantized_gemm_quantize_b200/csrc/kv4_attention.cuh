// Decode attention over a 4-bit KV cache, and the quantizer that writes it.
//
// The 4-bit KV cache of W4A8KV4 serving ("QServe/QoQ" abstract on the
// lmdeploy issue "[Feature] Support W4A8KV4 Quantization(QServe/QoQ)",
// Motivation: 4-bit KV cache, fused attention made memory-bound; "PrefixQuant
// ...", Key Findings: W4A4KV4). Format: one cached vector (a token of one kv
// head, D = 128 values) is quantized on its range widened to include zero,
// lo = min(min x, 0), hi = max(max x, 0): s = fp16_rn((hi - lo) / 15),
// z = clamp(rint(-lo / s), 0, 15), code = clamp(rint(x / s) + z, 0, 15)
// (fp32, IEEE divides, ties to even; s == 0 gives z = 0 and zero codes);
// codes two per byte (element 2i in bits 0-3 of byte i), 64 bytes per vector;
// (s, z) as one 32-bit word of two fp16 values, s in the low half.
//
// Decode attention: for sequence b (cache length L_b), query head h and its
// kv head g = h / (Hq / Hkv): s_j = scale * (s_j^K * sum_d q[d] (code - z)),
// o = sum_j softmax(s)_j (code^V_j - z^V_j) s^V_j, Y = fp16_rn(o). The cache is
// read once per four query heads: a CTA takes up to kKvChunk tokens of one
// (sequence, kv head) for up to four of its query heads, scores them,
// exponentiates against the chunk's own maximum and accumulates the weighted
// values; the last CTA of a (sequence, kv head, head group) to finish (a
// ticket in the workspace, no waiting) merges the chunks' partial results
// with exp(m_chunk - m) factors and writes Y. The scores and the weighted
// sums run on CUDA cores in fp32, about 14 operations per cache byte for four
// query heads per kv head, so at that grouping the arithmetic, not HBM, is
// expected to set the pace.
//
// Mapping inside a CTA (both phases): the chunk's K and V codes are staged in
// shared memory by two bulk copies issued at the start (all 2 x n x 64 bytes
// in flight at once); 8 lanes per token, lane slice li owns elements
// [16 li, 16 li + 16) (8 code bytes), so a warp reads 4 consecutive tokens =
// 256 contiguous bytes of shared memory per step. Products of an fp16 query
// element and a small integer (code - z) are exact in fp32.
#pragma once
#include "ptx.cuh"

namespace w4a8 {

constexpr int kKvD = 128;              // head dimension
constexpr int kKvRowBytes = kKvD / 2;  // packed codes of one cached vector
constexpr int kKvChunk = 256;          // tokens per CTA
constexpr int kKvThreads = 256;        // 8 warps
constexpr int kKvWarps = kKvThreads / 32;
constexpr int kErrKvRange = 7;         // W4A8_DEVERR_KV_RANGE
constexpr int kErrKvWait = 11;         // W4A8_DEVERR_KV_WAIT

// ------------------------------------------------------------ quantizer
struct KvQuantArgs {
  const __half* x;        // [n, 128] fp16 vectors
  int64_t n;
  uint8_t* codes;         // destination rows of 64 bytes
  uint32_t* params;       // destination (s, z) words
  const int32_t* pos;     // null: vector i -> row i; else vector i = b * H + h -> row (b * H + h) * Lmax + pos[b]
  int64_t H, Lmax;
  int* err;
};

// One warp per vector: lane l holds elements 4l .. 4l+3.
__global__ void __launch_bounds__(kKvThreads) kv4_quantize_kernel(KvQuantArgs a) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * kKvWarps;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kKvWarps + (threadIdx.x >> 5); i < a.n; i += warps) {
    int64_t row = i;
    if (a.pos != nullptr) {
      const int64_t b = i / a.H;
      const int p = a.pos[b];
      if (p < 0 || p >= a.Lmax) {  // the vector has no place in the cache: skipped and reported
        if (lane == 0) atomicCAS(a.err, 0, kErrKvRange);
        continue;
      }
      row = i * a.Lmax + p;
    }
    const uint2 raw = *reinterpret_cast<const uint2*>(a.x + i * kKvD + 4 * lane);
    const __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
    const __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
    const float v[4] = {__low2float(h01), __high2float(h01), __low2float(h23), __high2float(h23)};
    float lo = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
    float hi = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    lo = fminf(lo, 0.0f);
    hi = fmaxf(hi, 0.0f);
    const __half s = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
    const float sf = __half2float(s);
    // z and the codes as integers (rint half to even, then clamp): z is
    // stored as its integer's fp16 value, never a negative zero
    int zi = 0;
    uint32_t packed = 0;
    if (sf > 0.0f) {
      zi = min(max(__float2int_rn(__fdiv_rn(-lo, sf)), 0), 15);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = min(max(__float2int_rn(__fdiv_rn(v[e], sf)) + zi, 0), 15);
        packed |= static_cast<uint32_t>(c) << (4 * e);
      }
    }
    const float z = static_cast<float>(zi);
    reinterpret_cast<uint16_t*>(a.codes + row * kKvRowBytes)[lane] = static_cast<uint16_t>(packed);
    if (lane == 0) {
      const __half zh = __float2half_rn(z);
      a.params[row] = static_cast<uint32_t>(__half_as_ushort(s)) |
                      (static_cast<uint32_t>(__half_as_ushort(zh)) << 16);
    }
  }
}

// ------------------------------------------------------------ attention
struct KvAttnArgs {
  const __half* q;         // [B, Hq, 128]
  const uint8_t* kc;       // [B, Hkv, Lmax, 64]
  const uint32_t* kp;      // [B, Hkv, Lmax]
  const uint8_t* vc;
  const uint32_t* vp;
  const int32_t* seq_lens; // [B]
  __half* out;             // [B, Hq, 128]
  float* part;             // [B, Hq, nsplit, 2 + 128]: chunk max, chunk sum, weighted values
  int32_t* tickets;        // [B, Hkv, Hq / Hkv / GC], zero between launches
  int Hq, Hkv, nsplit;
  int64_t Lmax;
  float scale;
  int* err;
};

// (code - z) for the 16 codes of an 8-byte slice, exact: the code is placed
// in the mantissa of 2^23 (0x4B000000 | c = 2^23 + c) and 2^23 + z subtracted.
__device__ __forceinline__ void kv_unpack16(uint2 w, float bias, float (&x)[16]) {
  const uint32_t ww[2] = {w.x, w.y};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[8 * k + e] = __uint_as_float(0x4B000000u | ((ww[k] >> (4 * e)) & 0xFu)) - bias;
  }
}

__device__ __forceinline__ void kv_param(uint32_t p, float& s, float& bias) {
  s = __half2float(__ushort_as_half(static_cast<unsigned short>(p & 0xFFFFu)));
  bias = 8388608.0f + __half2float(__ushort_as_half(static_cast<unsigned short>(p >> 16)));
}

template <int GC>
__global__ void __launch_bounds__(kKvThreads) kv4_decode_kernel(KvAttnArgs a) {
  static_assert(GC == 1 || GC == 2 || GC == 4, "query heads per CTA");
  // the chunk's K and V codes, staged by two bulk copies (kKvChunk x 64 bytes
  // each); once the scores are done the K codes' space holds the per-warp
  // weighted values (s_o)
  constexpr int kKcBytes = kKvChunk * kKvRowBytes;
  constexpr int kOBytes = kKvWarps * GC * kKvD * 4;
  static_assert(kOBytes <= kKcBytes, "the weighted values fit in the K codes' space");
  __shared__ __align__(128) uint8_t s_kc[kKcBytes];
  __shared__ __align__(128) uint8_t s_vc[kKvChunk * kKvRowBytes];
  __shared__ float2 s_kpar[kKvChunk];  // per token: (s, 2^23 + z)
  __shared__ float2 s_vpar[kKvChunk];
  __shared__ uint64_t s_bar;
  __shared__ float s_q[GC][kKvD];
  __shared__ float s_p[GC][kKvChunk];
  __shared__ float s_m[GC], s_l[GC];
  float(*s_o)[GC][kKvD] = reinterpret_cast<float(*)[GC][kKvD]>(s_kc);
  __shared__ int s_last;

  const int split = blockIdx.x;
  const int hg = blockIdx.y;  // (kv head, head group)
  const int b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int groups = G / GC;
  const int g = hg / groups;
  const int h0 = g * G + (hg % groups) * GC;  // first query head of this CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 3, li = lane & 7;

  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_barrier_init();
  }
  grid_dependency_wait();  // q and the cache come from the preceding kernels
  grid_launch_dependents();

  int L = a.seq_lens[b];
  if (L < 0 || L > a.Lmax) {
    if (threadIdx.x == 0 && split == 0) atomicCAS(a.err, 0, kErrKvRange);
    L = L < 0 ? 0 : static_cast<int>(a.Lmax);
  }
  const int t0 = split * kKvChunk;
  const int n = max(0, min(L - t0, kKvChunk));  // tokens of this chunk
  const int64_t cache_row0 = (static_cast<int64_t>(b) * a.Hkv + g) * a.Lmax + t0;
  __syncthreads();  // the barrier is initialized
  // The chunk's codes are contiguous in the cache (64 bytes per token, rows
  // 64-byte aligned): two bulk copies put all of them in flight at once, so
  // the CTA streams its 2 x 16 KB instead of waiting once per token step.
  if (threadIdx.x == 0 && n > 0) {
    const uint64_t pol = l2_policy_evict_first();
    mbar_arrive_expect_tx(&s_bar, 2u * n * kKvRowBytes);
    bulk_load(s_kc, a.kc + cache_row0 * kKvRowBytes, n * kKvRowBytes, &s_bar, pol);
    bulk_load(s_vc, a.vc + cache_row0 * kKvRowBytes, n * kKvRowBytes, &s_bar, pol);
  }
  // parameter words (4 bytes per token: no 16-byte alignment to rely on) by plain loads
  for (int j = threadIdx.x; j < n; j += kKvThreads) {
    float sk, bk, sv, bv;
    kv_param(__ldg(a.kp + cache_row0 + j), sk, bk);
    kv_param(__ldg(a.vp + cache_row0 + j), sv, bv);
    s_kpar[j] = make_float2(sk, bk);
    s_vpar[j] = make_float2(sv, bv);
  }
  for (int i = threadIdx.x; i < GC * kKvD; i += kKvThreads)
    s_q[i / kKvD][i % kKvD] = __half2float(a.q[(static_cast<int64_t>(b) * a.Hq + h0 + i / kKvD) * kKvD + i % kKvD]);
  __syncthreads();
  if (n > 0 && !mbar_wait_limit(&s_bar, 0, nullptr, DevErr{a.err}, kErrKvWait, kWaitLimitNs)) {
    // the copies did not land in time (recorded): no result for this chunk
    // beyond zeros, and no exit while copies may still be in flight
    mbar_wait_limit(&s_bar, 0, nullptr, DevErr{a.err}, kErrKvWait, kWaitLimitNs);
  }

  // ---- scores: s_p[h][j] = scale * (s^K_j * sum_d q[d] (code - z))
  {
    float qr[GC][16];
#pragma unroll
    for (int h = 0; h < GC; ++h)
#pragma unroll
      for (int e = 0; e < 16; ++e) qr[h][e] = s_q[h][16 * li + e];
    for (int j0 = warp * 4; j0 < n; j0 += kKvWarps * 4) {
      const int j = j0 + grp;
      const bool valid = j < n;
      uint2 w = make_uint2(0u, 0u);
      float2 par = make_float2(0.0f, 8388608.0f);
      if (valid) {
        w = *reinterpret_cast<const uint2*>(s_kc + j * kKvRowBytes + li * 8);
        par = s_kpar[j];
      }
      const float sk = par.x, bias = par.y;
      float x[16];
      kv_unpack16(w, bias, x);
      float acc[GC];
#pragma unroll
      for (int h = 0; h < GC; ++h) {
        acc[h] = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[h] = fmaf(qr[h][e], x[e], acc[h]);
      }
#pragma unroll
      for (int h = 0; h < GC; ++h) {
        acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], 1);
        acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], 2);
        acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], 4);
      }
      if (valid && li == 0) {
#pragma unroll
        for (int h = 0; h < GC; ++h) s_p[h][j] = (sk * acc[h]) * a.scale;
      }
    }
  }
  __syncthreads();
  // ---- softmax over the chunk: warp h handles head h
  if (warp < GC) {
    float m = -INFINITY;
    for (int j = lane; j < n; j += 32) m = fmaxf(m, s_p[warp][j]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.0f;
    for (int j = lane; j < n; j += 32) {
      const float e = expf(s_p[warp][j] - m);
      s_p[warp][j] = e;
      l += e;
    }
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      s_m[warp] = m;
      s_l[warp] = l;
    }
  }
  __syncthreads();
  // ---- weighted values: lane (grp, li) sums its tokens for elements 16 li ..
  {
    float o[GC][16];
#pragma unroll
    for (int h = 0; h < GC; ++h)
#pragma unroll
      for (int e = 0; e < 16; ++e) o[h][e] = 0.0f;
    for (int j0 = warp * 4; j0 < n; j0 += kKvWarps * 4) {
      const int j = j0 + grp;
      if (j < n) {
        const uint2 w = *reinterpret_cast<const uint2*>(s_vc + j * kKvRowBytes + li * 8);
        const float sv = s_vpar[j].x, bias = s_vpar[j].y;
        float x[16];
        kv_unpack16(w, bias, x);
#pragma unroll
        for (int h = 0; h < GC; ++h) {
          const float wgt = s_p[h][j] * sv;
#pragma unroll
          for (int e = 0; e < 16; ++e) o[h][e] = fmaf(wgt, x[e], o[h][e]);
        }
      }
    }
    // the four token groups of the warp, then the warps
#pragma unroll
    for (int h = 0; h < GC; ++h)
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        o[h][e] += __shfl_xor_sync(0xffffffffu, o[h][e], 8);
        o[h][e] += __shfl_xor_sync(0xffffffffu, o[h][e], 16);
      }
    if (grp == 0) {
#pragma unroll
      for (int h = 0; h < GC; ++h)
#pragma unroll
        for (int e = 0; e < 16; ++e) s_o[warp][h][16 * li + e] = o[h][e];
    }
  }
  __syncthreads();
  // ---- this chunk's partial result
  const int64_t pstride = 2 + kKvD;
  for (int i = threadIdx.x; i < GC * kKvD; i += kKvThreads) {
    const int h = i / kKvD, d = i % kKvD;
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < kKvWarps; ++w) sum += s_o[w][h][d];
    float* pp = a.part + ((static_cast<int64_t>(b) * a.Hq + h0 + h) * a.nsplit + split) * pstride;
    pp[2 + d] = sum;
    if (d == 0) {
      pp[0] = s_m[h];
      pp[1] = n > 0 ? s_l[h] : 0.0f;
    }
  }
  // ---- the last chunk of this (sequence, head group) to finish merges them
  __threadfence();
  __syncthreads();
  int32_t* ticket = a.tickets + static_cast<int64_t>(b) * a.Hkv * groups + hg;
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1) == a.nsplit - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // Merge, in a fixed order (bit-reproducible): warp h finds head h's maximum
  // over the chunks that hold tokens and the denominator sum_c exp(m_c - m) l_c,
  // keeping the chunk factors exp(m_c - m) in shared memory (the spent V codes'
  // space); then every (head, element) thread sums its weighted values over the
  // chunks with independent loads.
  constexpr int kMergeSmem = kKcBytes / (4 * GC);  // chunk factors kept per head
  float* s_f = reinterpret_cast<float*>(s_vc);
  if (warp < GC) {
    const float* pp = a.part + (static_cast<int64_t>(b) * a.Hq + h0 + warp) * a.nsplit * pstride;
    float m = -INFINITY;
    for (int c = lane; c < a.nsplit; c += 32)
      if (__ldcg(pp + c * pstride + 1) > 0.0f) m = fmaxf(m, __ldcg(pp + c * pstride));
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float den = 0.0f;
    for (int c = lane; c < a.nsplit; c += 32) {
      const float lc = __ldcg(pp + c * pstride + 1);
      const float f = lc > 0.0f ? expf(__ldcg(pp + c * pstride) - m) : 0.0f;
      if (c < kMergeSmem) s_f[warp * kMergeSmem + c] = f;
      den = fmaf(f, lc, den);
    }
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) {
      s_m[warp] = m;
      s_l[warp] = den;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < GC * kKvD; i += kKvThreads) {
    const int h = i / kKvD, d = i % kKvD;
    const float* pp = a.part + (static_cast<int64_t>(b) * a.Hq + h0 + h) * a.nsplit * pstride;
    const float m = s_m[h], den = s_l[h];
    float num = 0.0f;
#pragma unroll 8
    for (int c = 0; c < a.nsplit; ++c) {
      float f;
      if (c < kMergeSmem) {
        f = s_f[h * kMergeSmem + c];
      } else {
        const float lc = __ldcg(pp + c * pstride + 1);
        f = lc > 0.0f ? expf(__ldcg(pp + c * pstride) - m) : 0.0f;
      }
      num = fmaf(f, __ldcg(pp + c * pstride + 2 + d), num);
    }
    a.out[(static_cast<int64_t>(b) * a.Hq + h0 + h) * kKvD + d] = __float2half_rn(den > 0.0f ? num / den : 0.0f);
  }
  if (threadIdx.x == 0) *ticket = 0;  // ready for the next launch
}

}  // namespace w4a8

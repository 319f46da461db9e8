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
// with exp(m_chunk - m) factors and writes Y. Both contractions (the scores
// and the weighted values) run on the tensor cores (tcgen05 kind::f16, fp32
// accumulation); the CUDA cores only unpack the codes (about one operation
// per code) and take the softmax. A CTA takes one chunk of 128 tokens, four
// CTAs share an SM; a second kernel merges the chunks of each (sequence,
// query head).
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace w4a8 {

constexpr int kKvD = 128;              // head dimension
constexpr int kKvRowBytes = kKvD / 2;  // packed codes of one cached vector
constexpr int kKvChunk = 128;          // tokens per CTA (one M = 128 tile)
constexpr int kKvThreads = 256;        // 8 warps (the quantizer)
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
  int B, Hq, Hkv, nsplit, groups;  // groups: head groups (of GC query heads) per kv head
  int64_t Lmax;
  float scale;
  int* err;
};

constexpr int kKvAttnThreads = 256;      // 8 warps: thread = (token, half of the head dimension)
constexpr int kKvPartStride = 2 + kKvD;  // floats per partial result

// Shared-memory layout of one attention CTA (offsets from a 1024-byte aligned
// base), sized for four CTAs per SM. The MMA operands built here use the
// 128-byte swizzle: within every 1024-byte atom of eight 128-byte rows, the
// 16-byte chunk c of row r sits at chunk position c ^ (r & 7).
struct KvSmem {
  static constexpr int kCodes = kKvChunk * kKvRowBytes;   // one matrix's codes of the chunk (8 KB)
  static constexpr int kPlane = kKvChunk * 128;           // 64 values x 2 bytes per token row
  static constexpr int kOpBlock = 16 * 128;               // one 64-column block of an N = 16 operand
  static constexpr int kOffVpl = 0;                       // V values, two planes (d 0-63, 64-127)
  static constexpr int kOffKc = kOffVpl + 2 * kPlane;     // K codes (bulk copy); later the weights
  static constexpr int kOffW = kOffKc;                    // (two blocks: tokens 0-63, 64-127)
  static constexpr int kOffVc = kOffKc + kCodes;          // V codes (bulk copy)
  static constexpr int kOffQ = kOffVc + kCodes;           // q: two blocks (d 0-63, 64-127)
  static constexpr int kOffScale = kOffQ + 2 * kOpBlock;  // per token (s^K, s^V)
  static constexpr int kOffZ = kOffScale + kKvChunk * 8;  // per token the z bits (K, V)
  static constexpr int kOffRed = kOffZ + kKvChunk * 4;    // [warp][head] max, then sum
  static constexpr int kOffMisc = kOffRed + 2 * 8 * 4 * 4;  // barriers, TMEM address, (m, l)
  static constexpr int kBytes = kOffMisc + 64 + 1024;       // + alignment slack
  static_assert(kOffKc % 1024 == 0 && kOffQ % 1024 == 0 && kOffW % 1024 == 0, "swizzle atoms 1024-aligned");
  static_assert(2 * kOpBlock <= kCodes, "the weights fit in the spent K codes");
  static_assert(kBytes + 1024 <= 232448 / 4, "four CTAs per SM");
};

// TMEM columns of one CTA: the dequantized K operand (64 columns of fp16
// pairs), the scores (16 fp32 columns) and the weighted values (16).
constexpr int kKvTmemK = 0, kKvTmemS = 64, kKvTmemO = 80, kKvTmemCols = 128;

// Position p (0..7) of an 8-value group of a dequantized row holds element
// kv_perm8(p) of the group: the unpacking below forms the pairs (e, e + 4)
// of the eight 4-bit codes of one 32-bit word.
__host__ __device__ constexpr int kv_perm8(int p) { return (p >> 1) + 4 * (p & 1); }

// (code - z) of the eight codes of word w as four fp16 pairs, exact: a code
// in bits 0-3 of a half goes into the mantissa of 1024 (0x6400 | c = 1024 +
// c) and bias = -(1024 + z) is added; one in bits 4-7 gives 1024 + 16 c,
// scaled by 1/16 in the fused multiply-add that adds bias16 = -(64 + z).
// Pair e holds elements (e, e + 4).
__device__ __forceinline__ void kv_unpack8_f16(uint32_t w, __half2 bias, __half2 bias16, uint32_t (&o)[4]) {
  const __half2 sixteenth = __float2half2_rn(0.0625f);
  const uint32_t w8 = w >> 8;
  const uint32_t x[4] = {(w & 0x000F000Fu) | 0x64006400u, (w & 0x00F000F0u) | 0x64006400u,
                         (w8 & 0x000F000Fu) | 0x64006400u, (w8 & 0x00F000F0u) | 0x64006400u};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __half2 h = *reinterpret_cast<const __half2*>(&x[e]);
    const __half2 v = (e & 1) ? __hfma2(h, sixteenth, bias16) : __hadd2(h, bias);
    o[e] = *reinterpret_cast<const uint32_t*>(&v);
  }
}
// The same as bf16 pairs (0x4300 | c = 128 + c; bf16 keeps 7 mantissa bits,
// so every code is shifted down to bits 0-3 first).
__device__ __forceinline__ void kv_unpack8_bf16(uint32_t w, __nv_bfloat162 bias, uint32_t (&o)[4]) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t x = ((w >> (4 * e)) & 0x000F000Fu) | 0x43004300u;
    const __nv_bfloat162 v = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&x), bias);
    o[e] = *reinterpret_cast<const uint32_t*>(&v);
  }
}

// Byte offset of element (row, col) of an N = 16 operand whose 64-column
// blocks are kOpBlock apart (16-bit elements, 128-byte swizzle).
__device__ __forceinline__ int kv_op_offset(int row, int col) {
  const int c = (col & 63) >> 3;
  return (col >> 6) * KvSmem::kOpBlock + row * 128 + ((c ^ (row & 7)) << 4) + ((col & 7) << 1);
}

// Decode attention on tensor cores. A CTA takes up to kKvChunk = 128 tokens
// of one (sequence, kv head) for GC of its query heads (a chunk without
// tokens only writes its empty partial result):
//  * the chunk's K and V codes arrive in shared memory by two bulk copies,
//    issued first;
//  * thread (token j, half hf) unpacks token j's K values of half hf, code -
//    z as fp16 (exact small integers), into TMEM lane j (the A operand of the
//    scores) and its V values as bf16 into row j of shared-memory plane hf;
//  * one thread issues S = K^ q^T: M = 128 tokens, N = 16 (the GC query
//    heads, fp16, the other rows zero), K = 128, fp32 accumulation: the
//    products of an fp16 query element and a small integer are exact;
//  * the threads read the scores of their token (heads hf, hf + 2),
//    s_j = scale * (s^K_j * S_j), take the chunk maximum and sum per head and
//    write the weights w_j = exp(s_j - m) s^V_j as three bf16 terms (w = t0 +
//    t1 + t2 up to 2^-24 relative: t0 = bf16(w), t1 = bf16(w - t0), t2 =
//    bf16(w - t0 - t1), the differences exact in fp32);
//  * one thread issues O = V^T W^T: M = 128 (the head dimension, V read
//    MN-major from the planes), N = 16 (three terms x GC heads), K = 128
//    tokens, products exact in fp32 (bf16 x small integer), fp32 sums;
//  * the threads read O, add the three terms of each head and write the
//    chunk's partial result (m, l, O); kv4_merge_kernel combines the chunks.
// The unpacking permutes each 8-value group of the head dimension
// (kv_perm8): q is staged in the same order, and row p of O is element
// 8 (p / 8) + kv_perm8(p % 8). Every wait is bounded.
template <int GC>
__global__ void __launch_bounds__(kKvAttnThreads, 4) kv4_decode_kernel(KvAttnArgs a) {
  static_assert(GC == 1 || GC == 2 || GC == 4, "query heads per CTA");
  extern __shared__ __align__(1024) uint8_t kv_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(kv_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_vpl = sm + KvSmem::kOffVpl;
  uint8_t* s_kc = sm + KvSmem::kOffKc;
  uint8_t* s_vc = sm + KvSmem::kOffVc;
  uint8_t* s_q = sm + KvSmem::kOffQ;
  uint8_t* s_w = sm + KvSmem::kOffW;
  float2* s_scale = reinterpret_cast<float2*>(sm + KvSmem::kOffScale);
  uint32_t* s_z = reinterpret_cast<uint32_t*>(sm + KvSmem::kOffZ);  // z bits: K low half, V high half
  float* s_rmax = reinterpret_cast<float*>(sm + KvSmem::kOffRed);   // [warp][head]
  float* s_rsum = s_rmax + 32;
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + KvSmem::kOffMisc);
  uint64_t* bar_mma = bar_ld + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_ld + 2);
  float* s_m = reinterpret_cast<float*>(s_tmem + 1);  // [4]
  float* s_l = s_m + 4;                               // [4]

  const int split = blockIdx.x;
  const int hg = blockIdx.y;  // (kv head, head group)
  const int b = blockIdx.z;
  const int g = hg / a.groups;
  const int h0 = g * (a.Hq / a.Hkv) + (hg % a.groups) * GC;  // first query head of this CTA
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int qd = warp & 3, hf = warp >> 2;  // TMEM lane quarter, half of the head dimension / head pair
  const int j = qd * 32 + lane;             // this thread's token (and TMEM lane)
  const DevErr err{a.err};

  grid_dependency_wait();  // q, the cache and the lengths come from the preceding kernels
  grid_launch_dependents();
  int L = __ldg(a.seq_lens + b);
  if (L < 0 || L > a.Lmax) {
    if (t == 0 && split == 0) atomicCAS(a.err, 0, kErrKvRange);
    L = L < 0 ? 0 : static_cast<int>(a.Lmax);
  }
  const int t0 = split * kKvChunk;
  const int n = max(0, min(L - t0, kKvChunk));  // tokens of this chunk
  const int64_t pbase = (static_cast<int64_t>(b) * a.Hq + h0) * a.nsplit + split;  // head h0's partial
  if (n == 0) {
    // no tokens: the empty partial result (m = -inf, l = 0, O = 0)
    for (int i = t; i < GC * kKvPartStride; i += kKvAttnThreads) {
      const int h = i / kKvPartStride, e = i % kKvPartStride;
      a.part[(pbase + static_cast<int64_t>(h) * a.nsplit) * kKvPartStride + e] = e == 0 ? -INFINITY : 0.0f;
    }
    return;
  }
  const int64_t cache_row0 = (static_cast<int64_t>(b) * a.Hkv + g) * a.Lmax + t0;
  if (t == 0) {
    // the chunk's codes are contiguous in the cache (64 bytes per token):
    // two bulk copies put all of them in flight before anything else
    mbar_init(bar_ld, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
    const uint64_t pol = l2_policy_evict_first();
    mbar_arrive_expect_tx(bar_ld, 2u * n * kKvRowBytes);
    bulk_load(s_kc, a.kc + cache_row0 * kKvRowBytes, n * kKvRowBytes, bar_ld, pol);
    bulk_load(s_vc, a.vc + cache_row0 * kKvRowBytes, n * kKvRowBytes, bar_ld, pol);
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, kKvTmemCols);
    tmem_relinquish();
  }
  // q's operand: rows 0..GC-1 the heads' queries in the unpack order of the
  // head dimension, the other rows zero
  for (int i = t; i < 2 * KvSmem::kOpBlock / 16; i += kKvAttnThreads)
    reinterpret_cast<uint4*>(s_q)[i] = make_uint4(0u, 0u, 0u, 0u);
  // per-token scales and z bits (plain loads: 4 bytes per token); tokens past
  // the chunk get s = 0, z = 0
  {
    const int jj = t & (kKvChunk - 1);
    const uint32_t* src = t < kKvChunk ? a.kp : a.vp;
    const uint32_t p = jj < n ? __ldg(src + cache_row0 + jj) : 0u;
    reinterpret_cast<float*>(s_scale)[2 * jj + (t < kKvChunk ? 0 : 1)] =
        __half2float(__ushort_as_half(static_cast<unsigned short>(p & 0xFFFFu)));
    reinterpret_cast<uint16_t*>(s_z)[2 * jj + (t < kKvChunk ? 0 : 1)] = static_cast<uint16_t>(p >> 16);
  }
  __syncthreads();  // zeroed before the queries are placed
  for (int i = t; i < GC * kKvD; i += kKvAttnThreads) {
    const int h = i / kKvD, p = i % kKvD;
    const int d = (p & ~7) + kv_perm8(p & 7);
    *reinterpret_cast<__half*>(s_q + kv_op_offset(h, p)) =
        a.q[(static_cast<int64_t>(b) * a.Hq + h0 + h) * kKvD + d];
  }
  tc_fence_before();
  __syncthreads();  // barriers, TMEM address, scales staged
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
  if (!mbar_wait_limit(bar_ld, 0, nullptr, err, kErrKvWait, kWaitLimitNs)) {
    // the copies did not land in time (recorded): no exit while they may
    // still be in flight
    mbar_wait_limit(bar_ld, 0, nullptr, err, kErrKvWait, kWaitLimitNs);
  }

  // ---- unpack: thread (token j, half hf); the K values first, so that the
  // scores' MMAs run while the V values are unpacked
  const uint32_t zz = s_z[j];
  const __half kz = __ushort_as_half(static_cast<unsigned short>(zz & 0xFFFFu));
  const __nv_bfloat16 vzb = __float2bfloat16_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(zz >> 16))));
  // the 32 code bytes of this half, read in an order that spreads the banks
  // (rows are 64 bytes: lanes two tokens apart share banks)
  const int rot = (j >> 1) & 1;
  const int base = j * kKvRowBytes + hf * 32;
  {
    const __half kb1 = __hadd(__float2half_rn(1024.0f), kz);
    const __half kb16 = __hadd(__float2half_rn(64.0f), kz);
    const __half2 kbias = __halves2half2(__hneg(kb1), __hneg(kb1));
    const __half2 kbias16 = __halves2half2(__hneg(kb16), __hneg(kb16));
    const uint4 ka = *reinterpret_cast<const uint4*>(s_kc + base + rot * 16);
    const uint4 kb = *reinterpret_cast<const uint4*>(s_kc + base + (rot ^ 1) * 16);
    const uint4 k0 = rot ? kb : ka, k1 = rot ? ka : kb;
    const uint32_t kws[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
    uint32_t kr[32];
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) {
      uint32_t o[4];
      kv_unpack8_f16(kws[wi], kbias, kbias16, o);
#pragma unroll
      for (int e = 0; e < 4; ++e) kr[4 * wi + e] = o[e];
    }
    tmem_st_32(tmem + kKvTmemK + 32 * hf + lane_base, kr);
  }
  tmem_wait_st();
  fence_proxy_async_smem();  // q's operand, before the MMAs read it
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (t == 0) {
    // S[token, head] = sum_d K^[token, d] q[head, d]
    constexpr uint32_t idesc = idesc_f16(128, 16);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t bdesc = smem_desc_k128_sw128(smem_u32(s_q) + (kk >> 2) * KvSmem::kOpBlock + (kk & 3) * 32);
      mma_f16_ts(tmem + kKvTmemS, tmem + kKvTmemK + kk * 8, bdesc, idesc, kk > 0 ? 1u : 0u);
    }
    mma_commit(bar_mma);
  }
  {
    const __nv_bfloat16 vb1 = __hadd(__float2bfloat16_rn(128.0f), vzb);
    const __nv_bfloat162 vbias = __halves2bfloat162(vb1, vb1);
    const uint4 vx = *reinterpret_cast<const uint4*>(s_vc + base + rot * 16);
    const uint4 vy = *reinterpret_cast<const uint4*>(s_vc + base + (rot ^ 1) * 16);
    const uint4 v0 = rot ? vy : vx, v1 = rot ? vx : vy;
    const uint32_t vws[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint8_t* row = s_vpl + hf * KvSmem::kPlane + j * 128;
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) {
      uint32_t o[4];
      kv_unpack8_bf16(vws[wi], vbias, o);
      *reinterpret_cast<uint4*>(row + ((wi ^ (j & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  fence_proxy_async_smem();  // the V planes, before the second MMAs read them (after the next barrier)
  if (!mbar_wait_limit(bar_mma, 0, nullptr, err, kErrKvWait, kWaitLimitNs))
    mbar_wait_limit(bar_mma, 0, nullptr, err, kErrKvWait, kWaitLimitNs);
  tc_fence_after();

  // ---- softmax over the chunk: thread (token j, heads hf and hf + 2)
  constexpr int kHp = GC >= 2 ? GC / 2 : 1;  // heads per thread
  const bool active = hf < GC;               // (GC == 1: the second half has no head)
  {
    uint32_t sv[16];
    tmem_ld_16_wait(tmem + kKvTmemS + lane_base, sv);
    const bool valid = j < n;
    const float2 sc = s_scale[j];
    float s[kHp], m[kHp], e[kHp];
#pragma unroll
    for (int k = 0; k < kHp; ++k) {
      const int h = hf + 2 * k;
      // column h = hf + 2k of the scores (selected without indexing by hf)
      const float sk = __uint_as_float(hf ? sv[(1 + 2 * k) & 3] : sv[(2 * k) & 3]);
      s[k] = (valid && active && h < GC) ? (sc.x * sk) * a.scale : -INFINITY;
      m[k] = s[k];
      for (int o = 16; o > 0; o >>= 1) m[k] = fmaxf(m[k], __shfl_xor_sync(0xffffffffu, m[k], o));
      if (lane == 0) s_rmax[warp * 4 + k] = m[k];
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kHp; ++k) {
      const int w0 = hf * 4;  // the four warps of this head pair
      m[k] = fmaxf(fmaxf(s_rmax[(w0 + 0) * 4 + k], s_rmax[(w0 + 1) * 4 + k]),
                   fmaxf(s_rmax[(w0 + 2) * 4 + k], s_rmax[(w0 + 3) * 4 + k]));
      e[k] = (valid && active) ? expf(s[k] - m[k]) : 0.0f;
      float l = e[k];
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) s_rsum[warp * 4 + k] = l;
    }
    // the weights w = e s^V as three bf16 terms: rows term * 4 + head of the
    // values' B operand, column = token (written over the spent K codes)
    if (active) {
#pragma unroll
      for (int k = 0; k < kHp; ++k) {
        const int h = hf + 2 * k;
        if (h >= GC) break;
        const float wt = e[k] * sc.y;
        const __nv_bfloat16 w0 = __float2bfloat16_rn(wt);
        const float r1 = wt - __bfloat162float(w0);
        const __nv_bfloat16 w1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 w2 = __float2bfloat16_rn(r1 - __bfloat162float(w1));
        *reinterpret_cast<__nv_bfloat16*>(s_w + kv_op_offset(h, j)) = w0;
        *reinterpret_cast<__nv_bfloat16*>(s_w + kv_op_offset(4 + h, j)) = w1;
        *reinterpret_cast<__nv_bfloat16*>(s_w + kv_op_offset(8 + h, j)) = w2;
      }
    }
    // (rows of the weights' operand beyond the heads keep the spent codes:
    // they only reach columns of O that are not read)
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (t < GC) {
    const int k = t >> 1, w0 = (t & 1) * 4;  // head t: pair t & 1, slot t >> 1
    s_m[t] = fmaxf(fmaxf(s_rmax[(w0 + 0) * 4 + k], s_rmax[(w0 + 1) * 4 + k]),
                   fmaxf(s_rmax[(w0 + 2) * 4 + k], s_rmax[(w0 + 3) * 4 + k]));
    s_l[t] = (s_rsum[(w0 + 0) * 4 + k] + s_rsum[(w0 + 1) * 4 + k]) +
             (s_rsum[(w0 + 2) * 4 + k] + s_rsum[(w0 + 3) * 4 + k]);
  }
  if (t == 0) {
    // O[d, n] = sum_token V^[token, d] W[n, token]: A = the V planes read
    // MN-major (64-value atoms along d: the second plane at +kPlane; 8-token
    // groups 1024 bytes apart), B = the weights, K-major
    constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (2u << 17) | (8u << 24);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t adesc = smem_desc_mn_sw128(smem_u32(s_vpl) + kk * 2048, KvSmem::kPlane, 1024);
      const uint64_t bdesc = smem_desc_k128_sw128(smem_u32(s_w) + (kk >> 2) * KvSmem::kOpBlock + (kk & 3) * 32);
      mma_f16_ss(tmem + kKvTmemO, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
    }
    mma_commit(bar_mma);
  }
  if (!mbar_wait_limit(bar_mma, 1, nullptr, err, kErrKvWait, kWaitLimitNs))
    mbar_wait_limit(bar_mma, 1, nullptr, err, kErrKvWait, kWaitLimitNs);
  tc_fence_after();

  // ---- the chunk's partial result: thread (output row j, heads hf, hf + 2)
  {
    uint32_t ov[16];
    tmem_ld_16_wait(tmem + kKvTmemO + lane_base, ov);
    const int d = (j & ~7) + kv_perm8(j & 7);
#pragma unroll
    for (int k = 0; k < kHp; ++k) {
      const int h = hf + 2 * k;
      if (h >= GC) break;
      float* pp = a.part + (pbase + static_cast<int64_t>(h) * a.nsplit) * kKvPartStride;
      const int c0 = 2 * k;  // columns term * 4 + h, selected without indexing by hf
      const float o0 = __uint_as_float(hf ? ov[c0 + 1] : ov[c0]);
      const float o1 = __uint_as_float(hf ? ov[4 + c0 + 1] : ov[4 + c0]);
      const float o2 = __uint_as_float(hf ? ov[8 + c0 + 1] : ov[8 + c0]);
      pp[2 + d] = (o0 + o1) + o2;
      if (j == 0) {
        pp[0] = s_m[h];
        pp[1] = s_l[h];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kKvTmemCols);
  }
}

// Merges the chunks' partial results of one (sequence, query head): m = max
// over the chunks that hold tokens, factors f_c = exp(m_c - m), den =
// sum_c f_c l_c, Y[d] = fp16_rn(sum_c f_c O_c[d] / den). One CTA per
// (sequence, head), thread d = element d; the factors of up to kMergeBlock
// chunks at a time are computed in parallel into shared memory, and every
// thread keeps 16 chunks' values in flight. Every sum runs in a fixed order
// (bit-reproducible).
constexpr int kMergeBlock = 1024;
__global__ void __launch_bounds__(kKvD) kv4_merge_kernel(KvAttnArgs a) {
  __shared__ float s_f[kMergeBlock];
  __shared__ float s_red[kKvD / 32];
  grid_dependency_wait();  // the partial results come from the preceding kernel
  grid_launch_dependents();
  const int h = blockIdx.x, b = blockIdx.y;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const float* pp = a.part + (static_cast<int64_t>(b) * a.Hq + h) * a.nsplit * kKvPartStride;
  // m over the chunks with tokens
  float m = -INFINITY;
  for (int c = t; c < a.nsplit; c += kKvD)
    if (pp[c * kKvPartStride + 1] > 0.0f) m = fmaxf(m, pp[c * kKvPartStride]);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  m = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
  __syncthreads();
  float den_part = 0.0f, num = 0.0f;
  constexpr int kBatch = 16;
  for (int c0 = 0; c0 < a.nsplit; c0 += kMergeBlock) {
    const int cn = min(kMergeBlock, a.nsplit - c0);
    for (int c = t; c < cn; c += kKvD) {
      const float lc = pp[(c0 + c) * kKvPartStride + 1];
      const float f = lc > 0.0f ? expf(pp[(c0 + c) * kKvPartStride] - m) : 0.0f;
      s_f[c] = f;
      den_part = fmaf(f, lc, den_part);
    }
    __syncthreads();
    for (int c1 = 0; c1 < cn; c1 += kBatch) {
      float v[kBatch];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) v[q] = c1 + q < cn ? pp[(c0 + c1 + q) * kKvPartStride + 2 + t] : 0.0f;
#pragma unroll
      for (int q = 0; q < kBatch; ++q)
        if (c1 + q < cn) num = fmaf(s_f[c1 + q], v[q], num);
    }
    __syncthreads();
  }
  for (int o = 16; o > 0; o >>= 1) den_part += __shfl_xor_sync(0xffffffffu, den_part, o);
  if (lane == 0) s_red[warp] = den_part;
  __syncthreads();
  const float den = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
  a.out[(static_cast<int64_t>(b) * a.Hq + h) * kKvD + t] = __float2half_rn(den > 0.0f ? num / den : 0.0f);
}

}  // namespace w4a8

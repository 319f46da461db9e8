// W4A8 GEMM on 5th-generation tensor cores (tcgen05, kind::i8), sm_100a.
//
//   Y[m, n] = fp16_rn( float(acc[m, n]) * (float(sA[m]) * float(s1[n])) )
//   acc[m, n] = sum_k A8[m, k] * W8[n, k],   W8 = (q - z) * s2  (exact int8)
//
// This is the W4A8 GEMM of the "QServe/QoQ" abstract (4-bit weights, 8-bit
// activations, progressive quantization so that dequantization is cheap) and
// of "LiquidGEMM: Hardware-Efficient W4A8 GEMM Kernel ..." (Method:
// overflow-free dequantization with two arithmetic operations per four
// elements, and weight load, dequantization and MMA overlapped in one
// pipeline without software synchronization in the hot loop).
//
// Structure: one persistent CTA per SM; warp-specialized roles that
// synchronize only through mbarriers (every wait bounded in time, reported
// through the device error word):
//   weight producer      one thread: per chunk of up to KS k-blocks of a
//                        tile, one 1-D bulk copy of the contiguous packed
//                        tiles (KS x 8320 bytes) into a weight ring slot;
//                        it starts before the dependency wait because the
//                        weights do not come from the preceding kernel.
//   activation producer  one thread: TMA 2-D loads of the int8 activation
//                        tiles (BN tokens x 128 k, 128-byte swizzle), after
//                        the programmatic-launch dependency wait.
//   dequantizers         DQ warpgroups; thread r owns weight row r of a tile:
//                        it reads its 64 code bytes as four 16-byte vectors
//                        and turns every four codes into four unsigned bytes
//                        W8 + 128 = q * s2 + (128 - z * s2) in [8, 248] with
//                        one AND and one IMAD (no carry crosses a byte), then
//                        writes them straight into tensor memory
//                        (tcgen05.st). The dequantized weights never touch
//                        shared memory (the point of the "QUICK" abstract's
//                        interleaving, reached here through TMEM).
//   MMA issuers          NMMA threads, alternate chunks:
//                        tcgen05.mma.kind::i8 with A = the dequantized
//                        weights in TMEM (u8, M = 128 rows = n), B = the
//                        activation tile in shared memory (s8, N = BN
//                        tokens), K = 32 per instruction; int32 accumulators
//                        in TMEM; both issuers accumulate into the same
//                        buffer (exact integer sums do not depend on order).
//   epilogue             four warps: tcgen05.ld of the accumulator, which it
//                        zeroes for its next use, minus 128 * rowsum[m]
//                        (undoes the weight bias exactly), scale, fp16 store
//                        (16-byte stores through a shared-memory transpose).
//
#pragma once
#include "pack.cuh"
#include "ptx.cuh"

namespace w4a8 {

struct GemmArgs {
  const uint8_t* tiles;  // packed weight tiles (blob + header)
  const __half* s1;      // per-output-channel scales (inside the blob)
  const __half* sA;      // per-token scales [M]
  const int32_t* rowsum; // per-token sums of the int8 activation codes [M]
  __half* Y;             // [M, N] fp16 (unused when acc_out != nullptr)
  int32_t* acc_out;      // optional: raw int32 accumulators [M, N]
  int32_t* ws_acc;       // [M, N] int32 partial sums: zero on entry and exit
  int32_t* ws_cnt;       // [num_tiles] tickets: zero on entry and exit
  int* err;              // device error word
  int M, N, KB;
  int m_tiles, num_tiles;
  int sk_tiles;          // the first sk_tiles tiles are split stream-K over all CTAs
  int split;             // > 1: cluster split-K, `split` CTAs (one cluster) per tile
  int band;              // whole tiles walk bands of `band` token tiles, channels fastest (0: no bands)
  int a4;                // activation codes are 4-bit, two per byte (W4A4), unpacked in shared memory
  const __half* lut_table;  // lookup-table weights: the 16 fp16 table entries (inside the blob)
};

struct Seg {
  int tile, kb0, kb1;
};

// The same deterministic schedule is replayed by every role of a CTA. Two
// kinds of work:
//   stream-K     the first sk_tiles tiles, flattened to (tile, k-block)
//                units: CTA i takes the i-th of grid equal ranges (its first
//                and last tiles are usually partial, reduced through the
//                global workspace);
//   whole tiles  the remaining tiles round robin, all k-blocks each.
// A CTA does its stream-K range first, so that the reduction of partial
// tiles overlaps the mainloop of its whole tiles and the last epilogue is a
// direct one. With cluster split-K instead, tile t is split into `split`
// k-ranges taken by the CTAs of cluster t (CTA rank r takes k-blocks
// [KB r / split, KB (r + 1) / split)) and reduced on chip.
// Whole tiles with band > 0 (and no stream-K tiles) are visited in bands of
// `band` token tiles: within a band the token tile changes fastest, then the
// channel tile, so that the CTAs running at one time share a band's
// activation rows (band x 128 rows x K bytes) in L2 instead of sweeping all
// of them once per channel column (tile index = channel tile x m_tiles +
// token tile throughout).
struct Sched {
  int64_t u, u_end;
  int tile_it, KB, num_tiles, split, band, m_tiles;
  __device__ __forceinline__ void init(const GemmArgs& a) {
    KB = a.KB;
    num_tiles = a.num_tiles;
    split = a.split;
    band = a.sk_tiles == 0 ? a.band : 0;
    m_tiles = a.m_tiles;
    u = u_end = 0;
    if (split > 1) {
      tile_it = static_cast<int>(blockIdx.x) / split;
      return;
    }
    if (a.sk_tiles > 0) {
      const int64_t U = static_cast<int64_t>(a.sk_tiles) * KB;
      u = U * blockIdx.x / gridDim.x;
      u_end = U * (blockIdx.x + 1) / gridDim.x;
    }
    tile_it = a.sk_tiles + static_cast<int>(blockIdx.x);
  }
  __device__ __forceinline__ bool next(Seg& s) {
    if (split > 1) {
      if (tile_it < 0 || tile_it >= num_tiles) return false;
      const int r = static_cast<int>(blockIdx.x) % split;
      s.tile = tile_it;
      s.kb0 = KB * r / split;
      s.kb1 = KB * (r + 1) / split;
      tile_it = -1;
      return true;
    }
    if (u < u_end) {
      s.tile = static_cast<int>(u / KB);
      s.kb0 = static_cast<int>(u - static_cast<int64_t>(s.tile) * KB);
      const int64_t left = u_end - u;
      s.kb1 = left < static_cast<int64_t>(KB - s.kb0) ? s.kb0 + static_cast<int>(left) : KB;
      u += s.kb1 - s.kb0;
      return true;
    }
    if (tile_it >= num_tiles) return false;
    s.tile = tile_it;
    if (band > 0 && band < m_tiles) {
      const int n_tiles = num_tiles / m_tiles;
      const int per_band = band * n_tiles;
      const int b = tile_it / per_band;               // bands before the last are full
      const int bm = min(band, m_tiles - b * band);  // token tiles of this band
      const int r = tile_it - b * per_band;
      s.tile = (r / bm) * m_tiles + b * band + r % bm;
    }
    s.kb0 = 0;
    s.kb1 = KB;
    tile_it += gridDim.x;
    return true;
  }
};

// Lookup-table weight tiles (weight-only GEMM, "Fast Matrix Multiplications
// for Lookup Table-Quantized LLMs"): 8192 index bytes + 128 fp16 row scales.
constexpr int kLutTileBytes = kTileCodeBytes + 2 * kTileN;  // 8448
// 3-bit lookup-table tiles: per row three 16-byte bit planes (plane c holds
// bit c of the row's 128 indices), plane c of row r at (c * 128 + r) * 16,
// then the 128 fp16 row scales.
constexpr int kLut3CodeBytes = 3 * 16 * kTileN;             // 6144
constexpr int kLut3TileBytes = kLut3CodeBytes + 2 * kTileN;  // 6400

template <int BN_, int KS_, int NS_, int NT_, int DQ_, int NACC_, int NMMA_, int LUT_ = 0, int MINB_ = 1>
struct GemmCfg {
  static constexpr int BN = BN_, KS = KS_, NS = NS_, NT = NT_, DQ = DQ_, NACC = NACC_, NMMA = NMMA_;
  // CTAs meant to be resident per SM (the register budget the compiler gets)
  static constexpr int kMinBlocks = MINB_;
  // LUT_ != 0: lookup-table weights against fp16 activations (kind::f16 MMA,
  // fp32 accumulators), 4-bit indices (1) or 3-bit indices in bit planes (3);
  // otherwise two-level 4-bit weights against int8 (kind::i8)
  static_assert(LUT_ == 0 || LUT_ == 1 || LUT_ == 3, "weight format");
  static constexpr bool kLut = LUT_ != 0;
  static constexpr bool kLut3 = LUT_ == 3;
  static constexpr int kTileB = kLut ? (kLut3 ? kLut3TileBytes : kLutTileBytes) : kTileBytes;  // one weight tile
  static constexpr int kKbCols = kLut ? 64 : 32;                    // TMEM columns of one dequantized k-block
  static constexpr int kMmaPerKb = kLut ? 8 : 4;                    // MMAs per k-block (K = 16 / 32)
  // pair table, one copy per lane: 256 entries (a byte of two 4-bit indices)
  // or 64 (a 6-bit pair code assembled from the three planes)
  static constexpr int kLutTableBytes = kLut ? (kLut3 ? 64 : 256) * 32 * 4 : 0;
  // One CTA per SM, persistent. Work moves in chunks of up to KS k-blocks of
  // one tile (one weight copy, one wait and one commit per chunk amortize the
  // fixed latencies of the synchronization operations).
  //   warp 0        weight producer (one thread) and TMEM owner
  //   warps 1..     NMMA MMA issuers (one thread each), chunk c goes to
  //                 issuer c % NMMA; both accumulate into the segment's one
  //                 accumulator buffer. With two issuers one thread's
  //                 barrier waits and commits overlap the other's MMAs, so
  //                 the tensor pipe does not idle between chunks when the
  //                 MMAs are thin (small BN).
  //   warp 1 lane 0 also issues the first kStartChunks weight copies at
  //                 kernel entry, before the rest of the set-up
  //   warp 3        activation producer (one thread)
  //   warps 4..     DQ dequantizer warpgroups, chunk c goes to group c % DQ
  //   last 4 warps  epilogue
  // Three rings: weight slots (NS, freed as soon as the dequantizers have
  // read them), activation slots (NS, freed when the chunk's MMAs finish)
  // and TMEM weight slots (NT, KS x 32 columns each, freed likewise).
  static constexpr int kDqWarp0 = 4;
  static constexpr int kEpWarp0 = 4 + 4 * DQ;
  static constexpr int kThreads = 32 * (4 + 4 * DQ + 4);
  static constexpr int kA8Bytes = BN * (kLut ? 256 : 128);  // one k-block of activations
  static constexpr int kASlot = KS * kA8Bytes;
  static constexpr int kWSlot = KS * kTileB;                // KS consecutive packed tiles
  static_assert(NMMA == 1 || NMMA == 2, "one or two MMA issuers (warps 1 and 2)");
  // Launch overlap for the small-token (decode) configurations, whose
  // launches are short enough for start-up and hand-over latency to matter:
  // the first weight chunks are requested at kernel entry, and the next
  // kernel in the stream is released as soon as every weight byte of the
  // grid has been requested. The large-token configurations release it after
  // their last MMA and start the weight stream after the set-up (measured
  // faster for their long launches).
  static constexpr bool kEarlyStart = BN <= 32;
  // Weight chunks requested at kernel entry, before the set-up. None: the
  // weight stream starts after the set-up. Measured on the decode step: two
  // chunks at entry 203.0 us per step, one 204.4, none 201.1 (the activation
  // tile, requested after the dependency wait, lands sooner behind fewer
  // queued weight bytes); the whole ring at entry delayed every CTA's first
  // weight bytes by about 1 us.
  static constexpr int kStartChunks = 0;
  static constexpr int kTmemA = NACC * BN;  // accumulators first, then the TMEM weight ring
  static constexpr int kTSlotCols = KS * kKbCols;
  // tensor memory columns allocated (a power of two >= 32)
  static constexpr int kTmemCols = kTmemA + NT * kTSlotCols <= 256 ? 256 : 512;
  static_assert(kTmemA + NT * kTSlotCols <= kTmemCols, "tensor memory budget");
  static_assert(NS >= 2 && NT >= 2, "two slots per ring at least");
  // Chunk c goes to dequantizer group c % DQ and to MMA issuer c % NMMA, and
  // every ring barrier is waited on by phase parity. A parity wait is exact
  // only if the waiting thread itself waited on the slot's previous phase
  // (the barrier is then at most one phase ahead): were a slot shared by two
  // groups or two issuers, a thread could find it one phase behind, and the
  // wait would pass on the stale parity (a TMEM slot or an activation slot
  // read before it is written). So every slot of a ring belongs to one
  // dequantizer group and one issuer: each ring depth is a multiple of both.
  static_assert(NS % DQ == 0 && NT % DQ == 0, "ring depths a multiple of the dequantizer groups");
  static_assert(NS % NMMA == 0 && NT % NMMA == 0, "ring depths a multiple of the MMA issuers");
  static_assert(NS >= NT, "weight ring at least as deep as the TMEM ring");
  // With enough TMEM slots a group keeps a chunk's TMEM stores in flight
  // while it loads its next chunk (it publishes chunk c only when it starts
  // chunk c + DQ, which must not need a slot that chunk c + 1 still holds);
  // otherwise it completes them within the chunk.
  static constexpr bool kPipelinedStores = NT >= 2 * DQ && NT >= DQ + 2;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
  // Cluster split-K (small BN only): up to kMaxSplit CTAs per tile. The
  // owner of TMEM lane quarter q is cluster rank q % split; it receives the
  // other ranks' 32 x BN partial sums of that quarter into kRecvSlots slots
  // of 32 x BN int32 (column-major: word j * 32 + row), at most 4 of them
  // for any split <= 4 (split 3: rank 0 owns two quarters, two senders each).
  static constexpr int kMaxSplit = BN <= 32 ? 4 : 1;
  static constexpr int kRecvSlots = kMaxSplit > 1 ? 4 : 0;
  static constexpr int kRecvSlotBytes = 32 * BN * 4;
  static constexpr int kOffA8 = 0;                 // 1024-aligned activation slots
  static constexpr int kOffW = NS * kASlot;        // 16-aligned weight slots
  static constexpr int kOffRecv = kOffW + NS * kWSlot;
  static constexpr int kOffLut = (kOffRecv + kRecvSlots * kRecvSlotBytes + 15) / 16 * 16;
  static constexpr int kOffBar = kOffLut + kLutTableBytes;
  // + one receive barrier per lane quarter + one packed-activation barrier per slot
  static constexpr int kNumBars = 4 * NS + 2 * NT + 2 * NACC + 1 + 4 + NS;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // epilogue per-token operands (128 int32 + 128 float), then the store
  // transpose (1 KB per epilogue warp, read as 16-byte vectors: 16-aligned)
  static constexpr int kOffRows = (kOffMisc + 64 + 15) / 16 * 16;
  static constexpr int kOffYStage = kOffRows + 1024;
  static_assert(kOffYStage % 16 == 0, "16-byte aligned store stage");
  static constexpr int kSmemBytes = kOffYStage + 4096 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

enum : int {
  kErrProducer = 1,
  kErrMma = 2,
  kErrDequant = 3,
  kErrEpilogue = 4,
  kErrDrain = 5,
};

// Dequantizes this thread's row r of a 128 x 128 weight tile in shared
// memory into 32 registers: register c holds the weights of k = 4c .. 4c+3
// (byte j = k 4c+j), the column order of the TMEM A operand, each as the
// unsigned byte W8 + 128 = q*s2 + (128 - z*s2) in [8, 248]: two integer
// operations per four weights (AND + IMAD; the high nibbles need one shift
// more), and no carry crosses a byte. The MMA reads them as u8 against s8
// activations; the epilogue removes the offset with 128 * rowsum.
__device__ __forceinline__ void dequant_tile_regs(const uint8_t* wt, int r, uint32_t (&out)[32]) {
  const uint32_t meta = wt[kTileCodeBytes + r];
  const uint32_t zq = meta & 15u, s2 = (meta >> 4) + 1u;
  const uint32_t bias = (128u - zq * s2) * 0x01010101u;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(wt + (c * kTileN + r) * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      out[c * 8 + 2 * jj] = (w[jj] & 0x0F0F0F0Fu) * s2 + bias;
      out[c * 8 + 2 * jj + 1] = ((w[jj] >> 4) & 0x0F0F0F0Fu) * s2 + bias;
    }
  }
}

// Dequantizes half h (in-tile k = 64h .. 64h+63) of row r of a lookup-table
// weight tile into 32 registers, register c holding the fp16 pair for
// k = 64h + 2c, 2c+1 (low half first, the column order of the TMEM A operand):
// W = fp16_rn(T[index] * s) by one 32-bit lookup of the pair table (entry e
// holds T[e & 15], T[e >> 4], the two indices of one byte) and one fp16x2
// multiply by the row's group scale s. The pair table has one copy per lane
// (entry e of copy l at word e * 32 + l, bank l), so a warp's lookups never
// conflict ("Fast Matrix Multiplications for Lookup Table-Quantized LLMs",
// abstract: vectorized and duplicated lookup table).
__device__ __forceinline__ void lut_dequant_half(const uint8_t* wt, int r, int h, const uint32_t* lut, int lane,
                                                 uint32_t (&out)[32]) {
  const __half sc = *reinterpret_cast<const __half*>(wt + kTileCodeBytes + 2 * r);
  const __half2 ss = __halves2half2(sc, sc);
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const uint4 v = *reinterpret_cast<const uint4*>(wt + ((2 * h + cc) * kTileN + r) * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t e = (w[jj] >> (8 * b)) & 0xFFu;
        const uint32_t pair = lut[e * 32 + lane];
        const __half2 x = __hmul2(*reinterpret_cast<const __half2*>(&pair), ss);
        out[cc * 16 + jj * 4 + b] = *reinterpret_cast<const uint32_t*>(&x);
      }
    }
  }
}

// The same for a 3-bit tile: index pair (k, k + 1), k even, is looked up by
// its 6-bit code f0 | f1 << 2 | f2 << 4, f_c = bits k, k + 1 of plane c (the
// pair table is built in that order), so a half reads two 32-bit words of
// each plane and needs no per-index bit gathering beyond the three fields.
__device__ __forceinline__ void lut3_dequant_half(const uint8_t* wt, int r, int h, const uint32_t* lut, int lane,
                                                  uint32_t (&out)[32]) {
  const __half sc = *reinterpret_cast<const __half*>(wt + kLut3CodeBytes + 2 * r);
  const __half2 ss = __halves2half2(sc, sc);
  const uint2 p0 = *reinterpret_cast<const uint2*>(wt + (0 * kTileN + r) * 16 + 8 * h);
  const uint2 p1 = *reinterpret_cast<const uint2*>(wt + (1 * kTileN + r) * 16 + 8 * h);
  const uint2 p2 = *reinterpret_cast<const uint2*>(wt + (2 * kTileN + r) * 16 + 8 * h);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const uint32_t a = j ? p0.y : p0.x, b = j ? p1.y : p1.x, c = j ? p2.y : p2.x;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t e = ((a >> (2 * i)) & 3u) | (((b >> (2 * i)) & 3u) << 2) | (((c >> (2 * i)) & 3u) << 4);
      const uint32_t pair = lut[e * 32 + lane];
      const __half2 x = __hmul2(*reinterpret_cast<const __half2*>(&pair), ss);
      out[j * 16 + i] = *reinterpret_cast<const uint32_t*>(&x);
    }
  }
}

// Accumulator words: int32 sums (biased, see store_output) or, for the
// lookup-table GEMM, fp32 bit patterns.
template <bool LUT>
__device__ __forceinline__ uint32_t acc_add(uint32_t a, uint32_t b) {
  if constexpr (LUT) {
    return __float_as_uint(__uint_as_float(a) + __uint_as_float(b));
  } else {
    return a + b;
  }
}

// Per-token operands of the epilogue, staged in shared memory per segment:
// thread t of the epilogue group loads token m0 + t before the group waits
// for the accumulator (one global load per thread, hidden behind the
// mainloop), and the store loops read them back as broadcast shared loads,
// so no global load sits between the accumulator and the output stores.
//
// Loads under a guard read an in-bounds address (the row is clamped, M >= 1)
// and let the guard only select the value. sA may be null (the accumulator
// output needs no scales): it is read with a plain load, never with the fp16
// __ldg overload, which is a side-effect-free asm statement that the compiler
// is free to evaluate ahead of the null test.
struct RowStage {
  int32_t* rowsum;  // [128]
  float* sa;        // [128]
  __device__ __forceinline__ void load(const GemmArgs& a, int m0, int t, int rows) {
    if (a.rowsum == nullptr) return;  // lookup-table GEMM: no per-token operands
    if (t < rows) {
      const int m = m0 + t;
      const int mc = m < a.M ? m : a.M - 1;
      const int32_t r = __ldg(a.rowsum + mc);
      float s = 0.0f;
      if (a.sA != nullptr) s = __half2float(a.sA[mc]);
      rowsum[t] = m < a.M ? r : 0;
      sa[t] = m < a.M ? s : 0.0f;
    }
  }
};

// Stores one output element: acc = biased sum - 128 * rowsum (exact in
// int32 for K <= 65536), then either the raw accumulator or
// fp16(acc * (sA * s1)).
__device__ __forceinline__ void store_output(const GemmArgs& a, int64_t o, uint32_t biased, int32_t rowsum, float sa,
                                             float s1f) {
  const int32_t acc = static_cast<int32_t>(biased - (static_cast<uint32_t>(rowsum) << 7));
  if (!in_bounds(o >= 0 && o < static_cast<int64_t>(a.M) * a.N, a.err)) return;
  if (a.acc_out != nullptr) {
    a.acc_out[o] = acc;
  } else {
    a.Y[o] = __float2half_rn(__fmul_rn(__int2float_rn(acc), __fmul_rn(sa, s1f)));
  }
}

// fp16 output of one element (no store): fp16(acc * (sA * s1)) with
// acc = biased sum - 128 * rowsum.
__device__ __forceinline__ __half output_half(uint32_t biased, int32_t rowsum, float sa, float s1f) {
  const int32_t acc = static_cast<int32_t>(biased - (static_cast<uint32_t>(rowsum) << 7));
  return __float2half_rn(__fmul_rn(__int2float_rn(acc), __fmul_rn(sa, s1f)));
}

// The same two for either kind of accumulator: the lookup-table GEMM's fp32
// sum is the output before rounding to fp16 (the scales were applied to the
// weights); the raw accumulator output holds its bit pattern.
template <bool LUT>
__device__ __forceinline__ void store_out(const GemmArgs& a, int64_t o, uint32_t v, int32_t rowsum, float sa,
                                          float s1f) {
  if constexpr (LUT) {
    if (!in_bounds(o >= 0 && o < static_cast<int64_t>(a.M) * a.N, a.err)) return;
    if (a.acc_out != nullptr) {
      a.acc_out[o] = static_cast<int32_t>(v);
    } else {
      a.Y[o] = __float2half_rn(__uint_as_float(v));
    }
  } else {
    store_output(a, o, v, rowsum, sa, s1f);
  }
}
template <bool LUT>
__device__ __forceinline__ __half out_half(uint32_t v, int32_t rowsum, float sa, float s1f) {
  if constexpr (LUT) {
    return __float2half_rn(__uint_as_float(v));
  } else {
    return output_half(v, rowsum, sa, s1f);
  }
}
template <bool LUT>
__device__ __forceinline__ void red_add_acc(int32_t* p, uint32_t v) {
  if constexpr (LUT) {
    red_add_f32(reinterpret_cast<float*>(p), __uint_as_float(v));
  } else {
    red_add_s32(p, static_cast<int32_t>(v));
  }
}

// Stores a warp's 16 rows x 32 channels of fp16 output (lane = channel
// n_base + lane, h[j] = row m_start + j) with 16-byte stores: the block is
// transposed through the warp's 1 KB shared-memory stage so that each
// instruction writes 8 whole 64-byte row pieces instead of 2 bytes a lane.
__device__ __forceinline__ void store_y_rows16(const GemmArgs& a, __half* stage, const __half (&h)[16], int m_start,
                                               int64_t n_base, int lane) {
#pragma unroll
  for (int j = 0; j < 16; ++j) stage[j * 32 + lane] = h[j];
  __syncwarp();
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int r = pass * 8 + (lane >> 2), q = lane & 3;
    const uint4 v = *reinterpret_cast<const uint4*>(stage + r * 32 + q * 8);
    const int m = m_start + r;
    if (m < a.M && in_bounds(m >= 0 && n_base >= 0 && n_base + q * 8 + 8 <= a.N, a.err))
      *reinterpret_cast<uint4*>(a.Y + static_cast<int64_t>(m) * a.N + n_base + q * 8) = v;
  }
  __syncwarp();  // the stage is reused by the next block
}

// Epilogue of one segment for the four warps of an epilogue group (128
// threads, named barrier 1). `tacc` is this warp's lane quarter at the
// first lane's accumulator; lane j's accumulator is `lane_stride * j`
// columns further; bit j of `lanes_used` says whether lane j holds a partial
// sum for this segment. Returns false if the group has to abort.
template <int BN, bool LUT>
__device__ __forceinline__ bool epilogue_segment(const GemmArgs& args, const Seg& sg, bool ok_in, uint64_t* accfull,
                                                 uint32_t bph, uint64_t* accempty, uint32_t tacc,
                                                 uint32_t lane_stride, uint32_t lanes_used, int quarter, int lane,
                                                 RowStage rows, __half* ystage, volatile int* abort_flag,
                                                 volatile int* epi_fail, volatile int* last_flag, DevErr err) {
  const int m_tile = sg.tile % args.m_tiles, n_tile = sg.tile / args.m_tiles;
  const int64_t N = args.N;
  const int64_t n = static_cast<int64_t>(n_tile) * kTileN + quarter * 32 + lane;
  const int m0 = m_tile * BN;
  const bool whole = (sg.kb0 == 0 && sg.kb1 == args.KB);
  const float s1f = LUT ? 1.0f : __half2float(args.s1[n]);
  named_bar_sync(1, 128);  // the previous segment's reads of the stage are done
  rows.load(args, m0, quarter * 32 + lane, BN);
  // the four warps take one decision, so every named barrier below is
  // reached by all of them
  bool ok = ok_in && mbar_wait(accfull, bph, abort_flag, err, kErrEpilogue);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && lane == 0) *epi_fail = 1;
  named_bar_sync(1, 128);
  if (*epi_fail) return false;
  tc_fence_after();
#pragma unroll 1
  for (int c = 0; c < BN; c += 16) {
    uint32_t v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = 0;
#pragma unroll 1
    for (uint32_t l = 0, used = lanes_used; used != 0; ++l, used >>= 1) {
      if (used & 1u) {
        uint32_t u[16];
        tmem_ld_16_wait(tacc + l * lane_stride + c, u);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = acc_add<LUT>(v[j], u[j]);
      }
    }
    tmem_zero_16(tacc + c);  // every MMA accumulates: the buffer starts the next segment at zero
    int32_t rsv[16];
    float sav[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      rsv[j] = rows.rowsum[c + j];
      sav[j] = rows.sa[c + j];
    }
    if (!whole) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int m = m0 + c + j;
        if (m < args.M && in_bounds(n < N && args.ws_acc != nullptr, args.err))
          red_add_acc<LUT>(args.ws_acc + static_cast<int64_t>(m) * N + n, v[j]);
      }
    } else if (args.acc_out != nullptr) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int m = m0 + c + j;
        if (m < args.M) store_out<LUT>(args, static_cast<int64_t>(m) * N + n, v[j], rsv[j], sav[j], s1f);
      }
    } else {
      __half h[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) h[j] = out_half<LUT>(v[j], rsv[j], sav[j], s1f);
      store_y_rows16(args, ystage, h, m0 + c, n - lane, lane);
    }
  }
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(accempty);
  if (!whole) {
    // Partial k-range: publish with red.add, then one thread releases the
    // group's writes and takes a ticket (bar.sync orders the other threads'
    // writes before its gpu-scope fence). The CTA whose ticket completes the
    // tile's k-blocks finishes the tile and restores the workspace to zero.
    named_bar_sync(1, 128);
    if (quarter == 0 && lane == 0) {
      const int add = sg.kb1 - sg.kb0;
      fence_acq_rel_gpu();
      const int old = in_bounds(sg.tile < args.num_tiles && args.ws_cnt != nullptr, args.err)
                          ? atom_add_relaxed_gpu(args.ws_cnt + sg.tile, add)
                          : -add;
      fence_acq_rel_gpu();
      *last_flag = (old + add == args.KB) ? 1 : 0;
    }
    named_bar_sync(1, 128);
    if (*last_flag) {
#pragma unroll 1
      for (int c = 0; c < BN; c += 16) {
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + c + j;
          const int mc = m < args.M ? m : args.M - 1;
          const uint32_t x = static_cast<uint32_t>(__ldcg(args.ws_acc + static_cast<int64_t>(mc) * N + n));
          v[j] = m < args.M ? x : 0u;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + c + j;
          if (m < args.M) {
            const int64_t o = static_cast<int64_t>(m) * N + n;
            __stcg(args.ws_acc + o, 0);
            store_out<LUT>(args, o, v[j], rows.rowsum[c + j], rows.sa[c + j], s1f);
          }
        }
      }
      if (quarter == 0 && lane == 0) args.ws_cnt[sg.tile] = 0;
    }
    named_bar_sync(1, 128);
  }
  return true;
}

// Epilogue of a cluster split-K tile for the four warps of the epilogue
// group: every CTA of the cluster holds the partial sums of its k-range; the
// owner of lane quarter q (rank q % split) receives the other ranks' 32 x BN
// partials of that quarter through distributed shared memory (st.async,
// counted by the owner's receive barrier), adds them and writes the rows.
template <class C>
__device__ __forceinline__ bool epilogue_cluster(const GemmArgs& args, const Seg& sg, uint64_t* accfull,
                                                 uint64_t* accempty, uint32_t tacc, uint32_t lanes_used,
                                                 int quarter, int lane, uint32_t* recv, uint64_t* recvbar,
                                                 RowStage rows, __half* ystage, volatile int* abort_flag,
                                                 volatile int* epi_fail, DevErr err) {
  constexpr int BN = C::BN;
  static_assert(BN <= 32, "one row block of per-token operands");
  const int m_tile = sg.tile % args.m_tiles, n_tile = sg.tile / args.m_tiles;
  const int64_t N = args.N;
  const int64_t n = static_cast<int64_t>(n_tile) * kTileN + quarter * 32 + lane;
  const int m0 = m_tile * BN;
  const float s1f = C::kLut ? 1.0f : __half2float(args.s1[n]);
  rows.load(args, m0, quarter * 32 + lane, BN);  // made visible by the barrier after the accumulator wait
  cluster_wait();                                // every receive barrier of the cluster is armed
  bool ok = mbar_wait(accfull, 0, abort_flag, err, kErrEpilogue);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && lane == 0) *epi_fail = 1;
  named_bar_sync(1, 128);
  if (*epi_fail) return false;
  tc_fence_after();
  uint32_t v[BN];
#pragma unroll
  for (int c = 0; c < BN; c += 16) {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[c + j] = 0;
#pragma unroll 1
    for (uint32_t l = 0, used = lanes_used; used != 0; ++l, used >>= 1) {
      if (used & 1u) {
        uint32_t u[16];
        tmem_ld_16_wait(tacc + l * BN + c, u);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[c + j] = acc_add<C::kLut>(v[c + j], u[j]);
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(accempty);

  const int S = args.split;
  const int rank = static_cast<int>(cluster_ctarank());
  const int owner = quarter % S;
  const int slot0 = (quarter / S) * (S - 1);  // this quarter's first receive slot at its owner
  if (owner != rank) {
    const int slot = slot0 + (rank < owner ? rank : rank - 1);
    const uint32_t dst = mapa_shared(smem_u32(recv) + slot * C::kRecvSlotBytes + lane * 4, owner);
    const uint32_t bar = mapa_shared(smem_u32(&recvbar[quarter]), owner);
#pragma unroll
    for (int j = 0; j < BN; ++j) st_async_b32(dst + j * 128, v[j], bar);
    return true;
  }
  ok = mbar_wait(&recvbar[quarter], 0, abort_flag, err, kErrEpilogue);
  if (!__all_sync(0xffffffffu, ok)) return false;
#pragma unroll 1
  for (int sidx = 0; sidx < S - 1; ++sidx) {
    const uint32_t* src = recv + (slot0 + sidx) * (C::kRecvSlotBytes / 4) + lane;
#pragma unroll
    for (int j = 0; j < BN; ++j) v[j] = acc_add<C::kLut>(v[j], src[j * 32]);
  }
  if (args.acc_out != nullptr) {
#pragma unroll
    for (int j = 0; j < BN; ++j) {
      const int m = m0 + j;
      if (m < args.M) store_out<C::kLut>(args, static_cast<int64_t>(m) * N + n, v[j], rows.rowsum[j], rows.sa[j], s1f);
    }
    return true;
  }
#pragma unroll
  for (int c = 0; c < BN; c += 16) {
    __half h[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) h[j] = out_half<C::kLut>(v[c + j], rows.rowsum[c + j], rows.sa[c + j], s1f);
    store_y_rows16(args, ystage, h, m0 + c, n - lane, lane);
  }
  return true;
}

// Four 4-bit two's complement codes (one per byte, bits 0-3) -> four int8.
__device__ __forceinline__ uint32_t sign_extend_nibbles(uint32_t x) {
  return x | ((x & 0x08080808u) * 0x1Eu);  // bit 3 set: OR 0xF0 into that byte (no carry leaves a byte)
}

// 16 packed 4-bit codes (8 bytes, code 2j in the low nibble of byte j) ->
// 16 int8 codes in k order.
__device__ __forceinline__ uint4 expand_codes4(uint2 p) {
  const uint32_t e0 = p.x & 0x0F0F0F0Fu, o0 = (p.x >> 4) & 0x0F0F0F0Fu;  // codes 0,2,4,6 / 1,3,5,7
  const uint32_t e1 = p.y & 0x0F0F0F0Fu, o1 = (p.y >> 4) & 0x0F0F0F0Fu;  // codes 8,.. / 9,..
  uint4 o;
  o.x = sign_extend_nibbles(__byte_perm(e0, o0, 0x5140));  // codes 0..3
  o.y = sign_extend_nibbles(__byte_perm(e0, o0, 0x7362));  // codes 4..7
  o.z = sign_extend_nibbles(__byte_perm(e1, o1, 0x5140));  // codes 8..11
  o.w = sign_extend_nibbles(__byte_perm(e1, o1, 0x7362));  // codes 12..15
  return o;
}

// Expands packed 4-bit activation codes [M, K/2] into int8 codes [M, K]
// (16 codes per thread and step, 8 bytes in, 16 out; HBM-bound). Used before
// the int8 GEMM when the token tiles are large: each activation tile is then
// expanded once instead of once per output tile.
__global__ void expand_act4_kernel(const uint2* __restrict__ packed, int64_t units, uint4* __restrict__ out) {
  grid_launch_dependents();  // the GEMM after this kernel may start its weight stream
  grid_dependency_wait();    // the codes come from the preceding kernel
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < units; i += stride)
    out[i] = expand_codes4(__ldcs(packed + i));
}

// Activation producer for 4-bit activations (W4A4, "PrefixQuant ...", Key
// Findings): the codes arrive packed, two per byte (64 bytes per token per
// k-block). Lane 0 loads each k-block's packed tile (BN rows x 64 bytes) by
// TMA into the upper half of its activation slot; the warp then expands it in
// place into the int8 layout the MMA reads (BN rows x 128 bytes, 128-byte
// swizzle: 16-byte piece c of row r at r * 128 + ((c ^ (r & 7)) * 16)) and
// releases the slot to the MMA issuers. Rows are expanded in ascending groups
// of four, in batches of up to eight groups; the packed bytes of every row a
// group overwrites have been read by then (group g writes bytes
// [512 g, 512 g + 512), which hold packed rows 8 g - BN .. 8 g - BN + 7 <=
// 4 g + 3), and all lanes read a batch before any lane writes it.
// The warp polls two conditions (non-blocking tests, with a short sleep when
// neither holds) and serves whichever is ready, expansion first: the oldest
// loaded chunk has arrived (expand it, in load order), or
// the slot of the next chunk is free (load it). A load never waits behind an
// expansion nor an expansion behind a free slot, so the loads run up to NS
// chunks ahead while every arrived chunk reaches the MMA at once. Neither
// wait can be part of a cycle: a slot frees when the MMAs of the chunk
// loaded NS chunks earlier finish, and that chunk was expanded before.
template <class C>
__device__ __forceinline__ void act4_producer(const GemmArgs& args, const CUtensorMap* tmap, uint8_t* sA8,
                                              uint64_t* afull, uint64_t* aempty, uint64_t* astage, int lane,
                                              volatile int* dep_done, volatile int* abort_flag, DevErr err) {
  constexpr int BN = C::BN, KS = C::KS, NS = C::NS;
  constexpr int kPackedRow = 64;  // bytes of one token's 128 codes
  grid_dependency_wait();         // the codes come from the preceding kernel
  if (lane == 0) *dep_done = 1;
  int cnt_ring[NS] = {};
  Sched sch;
  sch.init(args);
  Seg sg;
  bool have_seg = sch.next(sg);
  int kb = have_seg ? sg.kb0 : 0;
  int issued = 0, expanded = 0;
  bool ok = true;
  uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    bool progressed = false;
    if (expanded < issued) {
      const int a = expanded % NS;
      if (__all_sync(0xffffffffu, mbar_test_wait(smem_u32(&astage[a]), (expanded / NS) & 1))) {
        const int cnt = cnt_ring[a];
        for (int j = 0; j < cnt; ++j) {
          uint8_t* base = sA8 + a * C::kASlot + j * C::kA8Bytes;
          const uint8_t* packed = base + BN * kPackedRow;
          // batches of up to 8 row groups: all of a batch's packed bytes are
          // read (independent loads) before any of its rows is written
          constexpr int kGroups = BN / 4, kBatch = kGroups < 8 ? kGroups : 8;
          const int c = lane & 7;
#pragma unroll 1
          for (int g0 = 0; g0 < kGroups; g0 += kBatch) {
            uint2 p[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
              p[b] = *reinterpret_cast<const uint2*>(packed + (4 * (g0 + b) + (lane >> 3)) * kPackedRow + c * 8);
            __syncwarp();
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
              const int row = 4 * (g0 + b) + (lane >> 3);
              *reinterpret_cast<uint4*>(base + row * 128 + ((c ^ (row & 7)) << 4)) = expand_codes4(p[b]);
            }
            __syncwarp();
          }
        }
        fence_proxy_async_smem();  // the MMA (async proxy) reads what these generic stores wrote
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[a]);
        ++expanded;
        progressed = true;
      }
    }
    if (!progressed && have_seg) {
      const int a = issued % NS;
      if (__all_sync(0xffffffffu, mbar_test_wait(smem_u32(&aempty[a]), ((issued / NS) & 1) ^ 1))) {
        const int cnt = min(KS, sg.kb1 - kb);
        const int m0 = (sg.tile % args.m_tiles) * BN;
        if (lane == 0) {
          mbar_arrive_expect_tx(&astage[a], cnt * BN * kPackedRow);
          for (int j = 0; j < cnt; ++j)
            tma_load_2d(sA8 + a * C::kASlot + j * C::kA8Bytes + BN * kPackedRow, tmap, &astage[a],
                        (kb + j) * kPackedRow, m0);
        }
        cnt_ring[a] = cnt;
        ++issued;
        kb += KS;
        if (kb >= sg.kb1) {
          have_seg = sch.next(sg);
          if (have_seg) kb = sg.kb0;
        }
        progressed = true;
      }
    }
    if (!have_seg && expanded == issued) break;
    if (progressed) {
      t0 = global_timer_ns();
      continue;
    }
    // nothing ready: sleep briefly instead of spinning, which would take issue
    // slots from the dequantizer warps on this SM sub-partition
    __nanosleep(128);
    if ((it & 31u) == 0) {
      // nothing ready: the same bounds as every other wait of the kernel,
      // decided once for the whole warp
      if (__any_sync(0xffffffffu, *abort_flag != 0)) {
        ok = false;
        break;
      }
      const uint64_t now = global_timer_ns();
      bool expired = false;
      if (now < t0) {
        t0 = now;
      } else if (now - t0 > kWaitLimitNs) {
        expired = true;
      }
      if (__any_sync(0xffffffffu, expired)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicCAS(err.word, 0, kErrProducer);
        }
        ok = false;
        break;
      }
    }
  }
  (void)ok;
  // copies still in flight must land before the CTA exits
  for (int u = expanded; u < issued; ++u) mbar_wait(&astage[u % NS], (u / NS) & 1, nullptr, err, kErrDrain);
  __syncwarp();
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, C::kMinBlocks) w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                                                                    const GemmArgs args) {
  constexpr int BN = C::BN, KS = C::KS, NS = C::NS, NT = C::NT, DQ = C::DQ, NACC = C::NACC, NMMA = C::NMMA;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA8 = smem + C::kOffA8;
  uint8_t* sW = smem + C::kOffW;
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + C::kOffBar);  // weight slot loaded
  uint64_t* wempty = wfull + NS;                                     // weight slot read by the dequantizers
  uint64_t* afull = wempty + NS;                                     // activation slot loaded
  uint64_t* aempty = afull + NS;                                     // activation slot's MMAs finished
  uint64_t* tfull = aempty + NS;                                     // TMEM weight slot written
  uint64_t* tempty = tfull + NT;                                     // TMEM weight slot's MMAs finished
  uint64_t* accfull = tempty + NT;                                   // a segment's MMAs finished
  uint64_t* accempty = accfull + NACC;                               // epilogue has read the accumulator
  uint64_t* done = accempty + NACC;                                  // all MMAs finished
  uint64_t* recvbar = done + 1;                                      // cluster partials received, per quarter
  uint64_t* astage = recvbar + 4;                                    // packed 4-bit activations loaded
  uint32_t* recv = reinterpret_cast<uint32_t*>(smem + C::kOffRecv);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 2);
  volatile int* epi_fail = reinterpret_cast<volatile int*>(misc + 3);
  volatile int* dep_done = reinterpret_cast<volatile int*>(misc + 4);  // dependency wait passed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DevErr err{args.err, dep_done};

  if (warp == 1) {
    // Weight starter: the weights do not come from the preceding kernel, so
    // the first kStartChunks chunks' copies go out before the rest of the
    // set-up (barriers, tensor memory, the CTA barrier). The weight producer
    // skips these chunks.
    if (lane == 0) {
      for (int i = 0; i < NS; ++i) {
        mbar_init(&wfull[i], 1);
        mbar_init(&wempty[i], 4);
      }
      fence_barrier_init();
      fence_proxy_async_smem();
      const uint64_t pol_w = l2_policy_evict_first();
      Sched s0;
      s0.init(args);
      Seg g0;
      int c = 0;
      while (c < C::kStartChunks && s0.next(g0)) {
        const uint8_t* wsrc = args.tiles + static_cast<int64_t>(g0.tile / args.m_tiles) * args.KB * C::kTileB;
        for (int kb = g0.kb0; kb < g0.kb1 && c < C::kStartChunks; kb += KS, ++c) {
          const int cnt = min(KS, g0.kb1 - kb);
          mbar_arrive_expect_tx(&wfull[c], cnt * C::kTileB);
          bulk_load(sW + c * C::kWSlot, wsrc + static_cast<int64_t>(kb) * C::kTileB, cnt * C::kTileB, &wfull[c],
                    pol_w);
        }
      }
    }
    __syncwarp();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&afull[i], 1);
      mbar_init(&aempty[i], 1);
      mbar_init(&astage[i], 1);
    }
    for (int i = 0; i < NT; ++i) {
      mbar_init(&tfull[i], 4);
      mbar_init(&tempty[i], 1);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&accfull[i], NMMA);
      mbar_init(&accempty[i], 4);
    }
    mbar_init(done, NMMA);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&recvbar[q], 1);
      // armed once: completes when the other ranks' partials of quarter q land
      if (C::kMaxSplit > 1 && args.split > 1 && q % args.split == static_cast<int>(cluster_ctarank()))
        mbar_arrive_expect_tx(&recvbar[q], (args.split - 1) * C::kRecvSlotBytes);
    }
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;
    misc[4] = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if constexpr (C::kLut3) {
    // pair table: entry e = (T[lo], T[hi]) as fp16x2 with the indices' bits
    // c taken from bits 2c (lo) and 2c + 1 (hi) of e; one copy per lane
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + C::kOffLut);
    const uint16_t* T = reinterpret_cast<const uint16_t*>(args.lut_table);
    for (int i = threadIdx.x; i < 64 * 32; i += C::kThreads) {
      const int e = i >> 5;
      const int lo = (e & 1) | ((e >> 1) & 2) | ((e >> 2) & 4);
      const int hi = ((e >> 1) & 1) | ((e >> 2) & 2) | ((e >> 3) & 4);
      lut[i] = static_cast<uint32_t>(__ldg(T + lo)) | (static_cast<uint32_t>(__ldg(T + hi)) << 16);
    }
  } else if constexpr (C::kLut) {
    // pair table: entry e = (T[e & 15], T[e >> 4]) as fp16x2, one copy per lane
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + C::kOffLut);
    const uint16_t* T = reinterpret_cast<const uint16_t*>(args.lut_table);
    for (int i = threadIdx.x; i < 256 * 32; i += C::kThreads) {
      const int e = i >> 5;
      lut[i] = static_cast<uint32_t>(__ldg(T + (e & 15))) | (static_cast<uint32_t>(__ldg(T + (e >> 4))) << 16);
    }
  }
  if (warp == 0) {
    tmem_alloc(&misc[0], C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 3 && lane == 0) prefetch_tensormap(&tmap_a);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  // cluster split-K: the receive barriers are initialized before any CTA of
  // the cluster may store into this one (the epilogue waits on this phase)
  if (C::kMaxSplit > 1 && args.split > 1) cluster_arrive();

  Sched sch;
  sch.init(args);
  Seg sg;
  bool cluster_waited = false;

  if (warp == 0) {
    // ----------------------------------------------------- weight producer
    // The weights do not come from the preceding kernel, so they stream
    // without the dependency wait. One copy per chunk: the packed tiles of
    // consecutive k-blocks of a tile are contiguous. The first kStartChunks
    // chunks were issued by the weight starter at kernel entry.
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      int c = 0;
      bool ok = true;
      while (ok && sch.next(sg)) {
        const uint8_t* wsrc = args.tiles + static_cast<int64_t>(sg.tile / args.m_tiles) * args.KB * C::kTileB;
        for (int kb = sg.kb0; kb < sg.kb1; kb += KS, ++c) {
          if (c < C::kStartChunks) continue;
          const int cnt = min(KS, sg.kb1 - kb);
          const int w = c % NS;
          if (!mbar_wait(&wempty[w], ((c / NS) & 1) ^ 1, abort_flag, err, kErrProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&wfull[w], cnt * C::kTileB);
          bulk_load(sW + w * C::kWSlot, wsrc + static_cast<int64_t>(kb) * C::kTileB, cnt * C::kTileB, &wfull[w],
                    pol_w);
        }
      }
      // Every weight byte of this CTA is requested: the next kernel in the
      // stream may launch and start its own weight stream on the SMs this
      // grid frees (it waits for this grid to complete before it touches
      // anything this grid reads or writes).
      if (C::kEarlyStart) grid_launch_dependents();
      // copies still in flight must land before the CTA exits
      const int first = c - NS > 0 ? c - NS : 0;
      for (int i = first; i < c; ++i) mbar_wait(&wfull[i % NS], (i / NS) & 1, nullptr, err, kErrDrain);
    }
    __syncwarp();
  } else if (warp == 3 && args.a4) {
    // -------------------------------- activation producer, 4-bit activations
    if constexpr (!C::kLut) act4_producer<C>(args, &tmap_a, sA8, afull, aempty, astage, lane, dep_done, abort_flag, err);
  } else if (warp == 3) {
    // ------------------------------------------------- activation producer
    if (lane == 0) {
      grid_dependency_wait();  // the activation tiles come from the preceding kernel
      *dep_done = 1;           // the time limits of the CTA's waits start counting
      int c = 0;
      bool ok = true;
      while (ok && sch.next(sg)) {
        const int m0 = (sg.tile % args.m_tiles) * BN;
        for (int kb = sg.kb0; kb < sg.kb1; kb += KS, ++c) {
          const int cnt = min(KS, sg.kb1 - kb);
          const int a = c % NS;
          if (!mbar_wait(&aempty[a], ((c / NS) & 1) ^ 1, abort_flag, err, kErrProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&afull[a], cnt * C::kA8Bytes);
          for (int j = 0; j < cnt; ++j) {
            if constexpr (C::kLut) {
              // fp16 activations: a k-block is two 128-byte swizzle spans of 64 values
              tma_load_2d(sA8 + a * C::kASlot + j * C::kA8Bytes, &tmap_a, &afull[a], (kb + j) * 128, m0);
              tma_load_2d(sA8 + a * C::kASlot + j * C::kA8Bytes + BN * 128, &tmap_a, &afull[a], (kb + j) * 128 + 64,
                          m0);
            } else {
              tma_load_2d(sA8 + a * C::kASlot + j * C::kA8Bytes, &tmap_a, &afull[a], (kb + j) * 128, m0);
            }
          }
        }
      }
      const int first = c - NS > 0 ? c - NS : 0;
      for (int i = first; i < c; ++i) mbar_wait(&afull[i % NS], (i / NS) & 1, nullptr, err, kErrDrain);
    }
    __syncwarp();
  } else if (warp >= 1 && warp < 1 + NMMA) {
    // ----------------------------------------------------------- MMA issuers
    // Issuer mi takes chunks c = mi (mod NMMA) and with them whole ring slots
    // (depths are multiples of NMMA). Both issuers accumulate into
    // the segment's one accumulator buffer b: every MMA accumulates (the
    // epilogue hands the buffer back zeroed), so the order in which the tensor
    // pipe runs the two threads' MMAs does not change the exact int32 sums.
    // Each issuer commits every segment's accumulator barrier, with or without
    // MMAs of its own in that segment.
    if (lane == 0) {
      const int mi = warp - 1;
      constexpr uint32_t idesc = C::kLut ? idesc_f16(128, BN) : idesc_i8(128, BN);
      int c = 0, seg_i = 0;
      bool ok = true;
      while (ok && sch.next(sg)) {
        const int b = seg_i % NACC;
        if (!mbar_wait(&accempty[b], (seg_i / NACC) & 1, abort_flag, err, kErrMma)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + b * BN;
        for (int kb = sg.kb0; kb < sg.kb1; kb += KS, ++c) {
          if (c % NMMA != mi) continue;
          const int cnt = min(KS, sg.kb1 - kb);
          const int a = c % NS, t = c % NT;
          if (!mbar_wait(&tfull[t], (c / NT) & 1, abort_flag, err, kErrMma) ||
              !mbar_wait(&afull[a], (c / NS) & 1, abort_flag, err, kErrMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = tmem + C::kTmemA + t * C::kTSlotCols;
          const uint32_t b_addr = smem_u32(sA8 + a * C::kASlot);
          for (int j = 0; j < cnt; ++j) {
#pragma unroll
            for (int kk = 0; kk < C::kMmaPerKb; ++kk) {
              // each MMA consumes 32 bytes of every row of both operands (8
              // TMEM columns of A); fp16 activations span two swizzle atoms
              const uint32_t b_off = C::kLut ? (kk >> 2) * (BN * 128) + (kk & 3) * 32 : kk * 32;
              const uint64_t bdesc = smem_desc_k128_sw128(b_addr + j * C::kA8Bytes + b_off);
              if constexpr (C::kLut) {
                mma_f16_ts(d_tmem, a_tmem + j * C::kKbCols + kk * 8, bdesc, idesc, 1u);
              } else {
                mma_i8_ts(d_tmem, a_tmem + j * C::kKbCols + kk * 8, bdesc, idesc, 1u);
              }
            }
          }
          mma_commit(&aempty[a]);
          mma_commit(&tempty[t]);
        }
        if (!ok) break;
        mma_commit(&accfull[b]);
        ++seg_i;
      }
      // the next kernel in the stream may start its prologue now
      if (!C::kEarlyStart) grid_launch_dependents();
      // every issued MMA must finish before TMEM is released
      mma_commit(done);
      mbar_wait(done, 0, nullptr, err, kErrDrain);
    }
    __syncwarp();
  } else if (warp >= C::kDqWarp0 && warp < C::kDqWarp0 + 4 * DQ) {
    // --------------------------------------------------------- dequantizers
    // Group g takes chunks c = g (mod DQ). The weight slot is released as
    // soon as it has been read; with pipelined stores the TMEM stores of a
    // chunk stay in flight while the group loads and unpacks its next chunk.
    const int g = (warp - C::kDqWarp0) >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int c = 0, prev_t = -1;
    bool ok = true;
    while (ok && sch.next(sg)) {
      for (int kb = sg.kb0; kb < sg.kb1; kb += KS, ++c) {
        if (c % DQ != g) continue;
        const int cnt = min(KS, sg.kb1 - kb);
        const int w = c % NS, t = c % NT;
        // TMEM slot first, then the weight slot: both slots serve this group
        // alone (ring depths are multiples of DQ), so each parity wait is for
        // the phase after the one this group last waited on.
        if (!__all_sync(0xffffffffu, mbar_wait(&tempty[t], ((c / NT) & 1) ^ 1, abort_flag, err, kErrDequant) &&
                                         mbar_wait(&wfull[w], (c / NS) & 1, abort_flag, err, kErrDequant))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < cnt; ++j) {
          uint32_t out[32];
          if constexpr (C::kLut) {
            const uint32_t* lut = reinterpret_cast<const uint32_t*>(smem + C::kOffLut);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if constexpr (C::kLut3) {
                lut3_dequant_half(sW + w * C::kWSlot + j * C::kTileB, r, h, lut, lane, out);
              } else {
                lut_dequant_half(sW + w * C::kWSlot + j * C::kTileB, r, h, lut, lane, out);
              }
              if (C::kPipelinedStores && j == 0 && h == 0 && prev_t >= 0) {
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tfull[prev_t]);
              }
              tmem_st_32(tmem + C::kTmemA + t * C::kTSlotCols + j * C::kKbCols + h * 32 + lane_base, out);
            }
          } else {
            dequant_tile_regs(sW + w * C::kWSlot + j * C::kTileB, r, out);
            if (C::kPipelinedStores && j == 0 && prev_t >= 0) {
              // the previous chunk's stores are done once these ones may start
              tmem_wait_st();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tfull[prev_t]);
            }
            tmem_st_32(tmem + C::kTmemA + t * C::kTSlotCols + j * C::kKbCols + lane_base, out);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&wempty[w]);
        if (C::kPipelinedStores) {
          prev_t = t;
        } else {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tfull[t]);
        }
      }
    }
    tmem_wait_st();
    if (prev_t >= 0) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tfull[prev_t]);
    }
  } else if (warp >= C::kEpWarp0 && warp < C::kEpWarp0 + 4) {
    // ------------------------------------------------------------ epilogue
    // sA and rowsum come from the preceding kernel (the activation quantizer)
    grid_dependency_wait();
    const int quarter = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    RowStage rows{reinterpret_cast<int32_t*>(smem + C::kOffRows), reinterpret_cast<float*>(smem + C::kOffRows + 512)};
    __half* ystage = reinterpret_cast<__half*>(smem + C::kOffYStage + quarter * 1024);
    // every MMA accumulates: the accumulator buffers start at zero
    for (int b = 0; b < NACC; ++b)
      for (int c = 0; c < BN; c += 16) tmem_zero_16(tmem + b * BN + c + lane_base);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
      for (int b = 0; b < NACC; ++b) mbar_arrive(&accempty[b]);
    int seg_i = 0;
    while (sch.next(sg)) {
      const int b = seg_i % NACC;
      const uint32_t used = 1u;  // one accumulator per buffer
      if constexpr (C::kMaxSplit > 1) {
        if (args.split > 1) {
          // the single segment of a cluster split-K CTA
          cluster_waited = true;
          epilogue_cluster<C>(args, sg, &accfull[b], &accempty[b], tmem + b * BN + lane_base, used,
                              quarter, lane, recv, recvbar, rows, ystage, abort_flag, epi_fail, err);
          break;
        }
      }
      if (!epilogue_segment<BN, C::kLut>(args, sg, true, &accfull[b], (seg_i / NACC) & 1, &accempty[b],
                                tmem + b * BN + lane_base, BN, used, quarter, lane, rows, ystage,
                                abort_flag, epi_fail, last_flag, err))
        break;
      ++seg_i;
    }
  }

  // every thread of a cluster split-K launch waits on the cluster barrier
  // phase it arrived on (the epilogue group already has, unless it failed
  // before reaching it)
  __syncwarp();
  if (C::kMaxSplit > 1 && args.split > 1 && !__all_sync(0xffffffffu, cluster_waited)) cluster_wait();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace w4a8

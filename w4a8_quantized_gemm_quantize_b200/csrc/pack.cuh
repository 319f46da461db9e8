// Offline weight reordering into the GEMM's tile-native packed layout
// (compute-aware reordering of the codes, as in the "QServe/QoQ" abstract;
// offline interleaving so dequantized values never go back through shared
// memory, as in the "QUICK" abstract).
//
// Blob = 64-byte header, then (N/128) x (K/128) tiles of 8320 bytes, then s1.
// Tile (nt, kt) = 8192 code bytes + 128 meta bytes:
//   row r's codes for in-tile k = 8j .. 8j+7 form 32-bit word j: byte b has
//   k = 8j+b in its low nibble and k = 8j+4+b in its high nibble; word j of
//   row r is at word index ((j/4)*128 + r)*4 + j%4. So a thread owning row r
//   reads k = 32c .. 32c+31 as one 16-byte vector, a warp reads 512
//   contiguous bytes, and `w & 0x0F0F0F0F` / `(w >> 4) & 0x0F0F0F0F` yield
//   four consecutive k in the byte lanes of one register.
//   meta byte r = z | ((s2 - 1) << 4) for group kt.
// Header: u32 magic 'W4A8', u32 version 1, i64 N, i64 K, i32 group,
// u32 tile bytes, u64 byte offset of s1; zero elsewhere.
#pragma once
#include "ptx.cuh"

namespace w4a8 {

constexpr int kTileN = 128;
constexpr int kTileK = 128;
constexpr int kTileCodeBytes = kTileN * kTileK / 2;  // 8192
constexpr int kTileBytes = kTileCodeBytes + kTileN;  // 8320
constexpr int kHeaderBytes = 64;
constexpr uint32_t kMagic = 0x38413457u;  // "W4A8"
constexpr uint32_t kLayoutVersion = 1u;
// Device error code (W4A8_DEVERR_PACK_RANGE): a code or parameter outside its
// documented range reached a packer; the packed field keeps only its low bits.
constexpr int kErrPackRange = 8;

// One thread per (row n, 32-k chunk): 32 codes in, one 16-byte vector out.
__global__ void pack_codes_kernel(const uint8_t* __restrict__ q, int64_t N, int64_t K,
                                  uint8_t* __restrict__ tiles, int* err) {
  const int64_t KC = K >> 5;  // 32-k chunks per row
  const int64_t total = N * KC;
  const int64_t KT = K >> 7;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / KC;
    const int64_t kc = i - n * KC;  // global 32-chunk index
    const uint4* src = reinterpret_cast<const uint4*>(q + n * K + kc * 32);
    const uint4 a = src[0], b = src[1];
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};  // 4 codes per word, k ascending
    if (((a.x | a.y | a.z | a.w | b.x | b.y | b.z | b.w) & 0xF0F0F0F0u) != 0u) atomicCAS(err, 0, kErrPackRange);
    uint32_t out[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      // word for k = 8jj .. 8jj+7 of this chunk: low nibbles k..k+3, high k+4..k+7
      out[jj] = (in[2 * jj] & 0x0F0F0F0Fu) | ((in[2 * jj + 1] & 0x0F0F0F0Fu) << 4);
    }
    const int64_t nt = n >> 7, r = n & 127;
    const int64_t kt = kc >> 2, c = kc & 3;
    uint8_t* tile = tiles + (nt * KT + kt) * kTileBytes;
    *reinterpret_cast<uint4*>(tile + (c * kTileN + r) * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

__global__ void pack_meta_kernel(const uint8_t* __restrict__ z, const uint8_t* __restrict__ s2,
                                 const __half* __restrict__ s1, int64_t N, int64_t K, uint8_t* __restrict__ blob,
                                 int64_t s1_offset, int* err) {
  const int64_t G = K >> 7;
  const int64_t total = N * G;
  uint8_t* tiles = blob + kHeaderBytes;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / G, g = i - n * G;
    if (z[i] > 15 || s2[i] < 1 || s2[i] > 8) atomicCAS(err, 0, kErrPackRange);
    const uint8_t meta = static_cast<uint8_t>((z[i] & 0x0F) | (((s2[i] - 1) & 0x0F) << 4));
    tiles[((n >> 7) * G + g) * kTileBytes + kTileCodeBytes + (n & 127)] = meta;
  }
  __half* s1_out = reinterpret_cast<__half*>(blob + s1_offset);
  const int64_t s1_padded = ((2 * N + 15) / 16) * 8;  // in halves
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < s1_padded;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    s1_out[i] = i < N ? s1[i] : __ushort_as_half(0);
  }
  if (blockIdx.x == 0 && threadIdx.x < kHeaderBytes / 4) {
    uint32_t w = 0;
    switch (threadIdx.x) {
      case 0: w = kMagic; break;
      case 1: w = kLayoutVersion; break;
      case 2: w = static_cast<uint32_t>(N); break;
      case 3: w = static_cast<uint32_t>(static_cast<uint64_t>(N) >> 32); break;
      case 4: w = static_cast<uint32_t>(K); break;
      case 5: w = static_cast<uint32_t>(static_cast<uint64_t>(K) >> 32); break;
      case 6: w = 128u; break;
      case 7: w = static_cast<uint32_t>(kTileBytes); break;
      case 8: w = static_cast<uint32_t>(s1_offset); break;
      case 9: w = static_cast<uint32_t>(static_cast<uint64_t>(s1_offset) >> 32); break;
      default: w = 0; break;
    }
    reinterpret_cast<uint32_t*>(blob)[threadIdx.x] = w;
  }
}

// Lookup-table weight blob (weight-only GEMM, "Fast Matrix Multiplications
// for Lookup Table-Quantized LLMs", abstract: offline restructuring of the
// quantized weights). 64-byte header (u32 magic 'W4LT', u32 version 1,
// i64 N, i64 K, i32 group, u32 tile bytes 8448, u64 byte offset of the
// table), then (N/128) x (K/128) tiles of 8448 bytes, then the 16 fp16 table
// entries padded to 64 bytes. Tile (nt, kt) = 8192 index bytes + 128 fp16
// row scales of group kt: byte j of row r's 64 bytes holds the indices of
// in-tile k = 2j (bits 0-3) and k = 2j+1 (bits 4-7), so one pair-table
// lookup per byte yields two consecutive k; 16-byte vector c of the row is
// at (c * 128 + r) * 16 (a warp reads 512 contiguous bytes).
constexpr uint32_t kLutMagic = 0x544C3457u;  // "W4LT"
constexpr int kLutTileBytesPack = kTileCodeBytes + 2 * kTileN;  // 8448

// One thread per (row n, 32-k chunk): 32 indices in, one 16-byte vector out.
__global__ void lut_pack_codes_kernel(const uint8_t* __restrict__ q, int64_t N, int64_t K,
                                      uint8_t* __restrict__ tiles, int* err) {
  const int64_t KC = K >> 5;
  const int64_t total = N * KC;
  const int64_t KT = K >> 7;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / KC;
    const int64_t kc = i - n * KC;
    const uint4* src = reinterpret_cast<const uint4*>(q + n * K + kc * 32);
    const uint4 a = src[0], b = src[1];
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};  // 4 indices per word, k ascending
    if (((a.x | a.y | a.z | a.w | b.x | b.y | b.z | b.w) & 0xF0F0F0F0u) != 0u) atomicCAS(err, 0, kErrPackRange);
    uint32_t out[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      // 8 indices (k = 8jj .. 8jj+7 of the chunk) -> 4 bytes, pairs (2b, 2b+1)
      const uint32_t lo = in[2 * jj], hi = in[2 * jj + 1];
      const uint32_t e = __byte_perm(lo, hi, 0x6420) & 0x0F0F0F0Fu;  // indices k = 0, 2, 4, 6
      const uint32_t o = __byte_perm(lo, hi, 0x7531) & 0x0F0F0F0Fu;  // indices k = 1, 3, 5, 7
      out[jj] = e | (o << 4);
    }
    const int64_t nt = n >> 7, r = n & 127;
    const int64_t kt = kc >> 2, c = kc & 3;
    uint8_t* tile = tiles + (nt * KT + kt) * kLutTileBytesPack;
    *reinterpret_cast<uint4*>(tile + (c * kTileN + r) * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// Row scales into their tiles, the table after the tiles, and the header.
__global__ void lut_pack_meta_kernel(const __half* __restrict__ s, const __half* __restrict__ table, int64_t N,
                                     int64_t K, uint8_t* __restrict__ blob, int64_t table_offset) {
  const int64_t G = K >> 7;
  const int64_t total = N * G;
  uint8_t* tiles = blob + kHeaderBytes;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / G, g = i - n * G;
    *reinterpret_cast<__half*>(tiles + ((n >> 7) * G + g) * kLutTileBytesPack + kTileCodeBytes + 2 * (n & 127)) = s[i];
  }
  if (blockIdx.x == 0 && threadIdx.x < 32) {
    __half* t = reinterpret_cast<__half*>(blob + table_offset);
    t[threadIdx.x] = threadIdx.x < 16 ? table[threadIdx.x] : __ushort_as_half(0);
  }
  if (blockIdx.x == 0 && threadIdx.x < kHeaderBytes / 4) {
    uint32_t w = 0;
    switch (threadIdx.x) {
      case 0: w = kLutMagic; break;
      case 1: w = kLayoutVersion; break;
      case 2: w = static_cast<uint32_t>(N); break;
      case 3: w = static_cast<uint32_t>(static_cast<uint64_t>(N) >> 32); break;
      case 4: w = static_cast<uint32_t>(K); break;
      case 5: w = static_cast<uint32_t>(static_cast<uint64_t>(K) >> 32); break;
      case 6: w = 128u; break;
      case 7: w = static_cast<uint32_t>(kLutTileBytesPack); break;
      case 8: w = static_cast<uint32_t>(table_offset); break;
      case 9: w = static_cast<uint32_t>(static_cast<uint64_t>(table_offset) >> 32); break;
      default: w = 0; break;
    }
    reinterpret_cast<uint32_t*>(blob)[threadIdx.x] = w;
  }
}


// ------------------------------------------------ 3-bit lookup-table blob
// Tiles of 6400 bytes: per row three 16-byte bit planes (plane c = bit c of
// the row's 128 indices, bit kk of the plane = bit kk % 8 of byte kk / 8),
// plane c of row r at (c * 128 + r) * 16, then the 128 fp16 row scales; after
// the tiles the 8 fp16 table entries, zero padded to 64 bytes.
constexpr uint32_t kLut3Magic = 0x544C3357u;  // "W3LT"
constexpr int kLut3CodeBytesPack = 3 * 16 * kTileN;                 // 6144
constexpr int kLut3TileBytesPack = kLut3CodeBytesPack + 2 * kTileN;  // 6400

// One warp per (row n, tile column kt): lane l reads the index of in-tile
// k = 32w + l (w = 0..3), and a ballot of bit c gives word w of plane c.
__global__ void lut3_pack_codes_kernel(const uint8_t* __restrict__ q, int64_t N, int64_t K,
                                       uint8_t* __restrict__ tiles, int* err) {
  const int64_t KT = K >> 7;
  const int64_t total = N * KT;
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  for (int64_t i = blockIdx.x * wpb + (threadIdx.x >> 5); i < total; i += static_cast<int64_t>(gridDim.x) * wpb) {
    const int64_t n = i / KT, kt = i - n * KT;
    uint32_t w0[4], w1[4], w2[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t v = q[n * K + kt * 128 + 32 * w + lane];
      if (v > 7u) atomicCAS(err, 0, kErrPackRange);  // only bits 0-2 are packed
      w0[w] = __ballot_sync(0xffffffffu, (v & 1u) != 0);
      w1[w] = __ballot_sync(0xffffffffu, (v & 2u) != 0);
      w2[w] = __ballot_sync(0xffffffffu, (v & 4u) != 0);
    }
    uint8_t* tile = tiles + (n >> 7) * KT * kLut3TileBytesPack + kt * kLut3TileBytesPack;
    const int64_t r = n & 127;
    if (lane == 0) *reinterpret_cast<uint4*>(tile + (0 * kTileN + r) * 16) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
    if (lane == 1) *reinterpret_cast<uint4*>(tile + (1 * kTileN + r) * 16) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
    if (lane == 2) *reinterpret_cast<uint4*>(tile + (2 * kTileN + r) * 16) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
  }
}

// Row scales into their tiles, the table after the tiles, and the header.
__global__ void lut3_pack_meta_kernel(const __half* __restrict__ s, const __half* __restrict__ table, int64_t N,
                                      int64_t K, uint8_t* __restrict__ blob, int64_t table_offset) {
  const int64_t G = K >> 7;
  const int64_t total = N * G;
  uint8_t* tiles = blob + kHeaderBytes;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / G, g = i - n * G;
    *reinterpret_cast<__half*>(tiles + ((n >> 7) * G + g) * kLut3TileBytesPack + kLut3CodeBytesPack + 2 * (n & 127)) =
        s[i];
  }
  if (blockIdx.x == 0 && threadIdx.x < 32) {
    __half* t = reinterpret_cast<__half*>(blob + table_offset);
    t[threadIdx.x] = threadIdx.x < 8 ? table[threadIdx.x] : __ushort_as_half(0);
  }
  if (blockIdx.x == 0 && threadIdx.x < kHeaderBytes / 4) {
    uint32_t w = 0;
    switch (threadIdx.x) {
      case 0: w = kLut3Magic; break;
      case 1: w = kLayoutVersion; break;
      case 2: w = static_cast<uint32_t>(N); break;
      case 3: w = static_cast<uint32_t>(static_cast<uint64_t>(N) >> 32); break;
      case 4: w = static_cast<uint32_t>(K); break;
      case 5: w = static_cast<uint32_t>(static_cast<uint64_t>(K) >> 32); break;
      case 6: w = 128u; break;
      case 7: w = static_cast<uint32_t>(kLut3TileBytesPack); break;
      case 8: w = static_cast<uint32_t>(table_offset); break;
      case 9: w = static_cast<uint32_t>(static_cast<uint64_t>(table_offset) >> 32); break;
      default: w = 0; break;
    }
    reinterpret_cast<uint32_t*>(blob)[threadIdx.x] = w;
  }
}

}  // namespace w4a8

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
// Structure (one CTA per SM, persistent, 12 warps):
//   warp 0      producer: per k-block, a TMA 2-D load of the int8 activation
//               tile (BN tokens x 128 k, 128-byte swizzle) and a 1-D bulk
//               copy of the packed weight tile (128 n x 128 k, 8320 bytes)
//               into a STAGES-deep shared-memory ring.
//   warps 4-7   dequantizers: thread r of the warpgroup owns weight row r; it
//               reads its 64 code bytes as four 16-byte vectors and turns
//               every four codes into four int8 weights with
//               ((w & 0x0F0F0F0F) * s2 + (128 - z*s2) * 0x01010101) ^ 0x80808080
//               (each byte stays in [8, 248] before the xor, so no carry
//               crosses a byte), then writes the 128 int8 weights of its row
//               straight into tensor memory with tcgen05.st. The dequantized
//               weights never touch shared memory (the point of the "QUICK"
//               abstract's interleaving, reached here through TMEM).
//   warp 1      MMA issuer (one thread): tcgen05.mma.kind::i8 with A = the
//               dequantized weights in TMEM (M = 128 rows = n), B = the
//               activation tile in shared memory (N = BN tokens), K = 32 per
//               instruction; int32 accumulators in TMEM (two buffers).
//   warps 8-11  epilogue: tcgen05.ld of the accumulators (lane = n, column =
//               token), scale, fp16 store; or, for a partial k-range,
//               red.add into an int32 workspace and a ticket counter whose
//               last arriver finishes the tile (nobody spins on another CTA).
//   warp 2      owns the TMEM allocation.
// The roles synchronize only through mbarriers; every wait is bounded in
// time and reports through the device error word.
//
// Work split: tiles are (token block of BN) x (128 output channels), each
// with K/128 k-blocks. Either whole tiles round-robin over the CTAs, or
// ("stream-K") each CTA takes one contiguous range of the flattened
// (tile, k-block) sequence, which balances small-M problems whose tile count
// is below the SM count.
#pragma once
#include "pack.cuh"
#include "ptx.cuh"

namespace w4a8 {

struct GemmArgs {
  const uint8_t* tiles;  // packed weight tiles (blob + header)
  const __half* s1;      // per-output-channel scales (inside the blob)
  const __half* sA;      // per-token scales [M]
  __half* Y;             // [M, N] fp16 (unused when acc_out != nullptr)
  int32_t* acc_out;      // optional: raw int32 accumulators [M, N]
  int32_t* ws_acc;       // [M, N] int32 partial sums: zero on entry and exit
  int32_t* ws_cnt;       // [num_tiles] tickets: zero on entry and exit
  int* err;              // device error word
  int M, N, KB;
  int m_tiles, num_tiles;
  int stream_k;
};

struct Seg {
  int tile, kb0, kb1;
};

// The same deterministic schedule is replayed by every role of a CTA.
struct Sched {
  int64_t u, u_end;
  int tile_it, KB, num_tiles, stream_k;
  __device__ __forceinline__ void init(const GemmArgs& a) {
    KB = a.KB;
    num_tiles = a.num_tiles;
    stream_k = a.stream_k;
    if (stream_k) {
      const int64_t U = static_cast<int64_t>(num_tiles) * KB;
      u = U * blockIdx.x / gridDim.x;
      u_end = U * (blockIdx.x + 1) / gridDim.x;
    } else {
      tile_it = blockIdx.x;
    }
  }
  __device__ __forceinline__ bool next(Seg& s) {
    if (stream_k) {
      if (u >= u_end) return false;
      s.tile = static_cast<int>(u / KB);
      s.kb0 = static_cast<int>(u - static_cast<int64_t>(s.tile) * KB);
      const int64_t left = u_end - u;
      s.kb1 = left < static_cast<int64_t>(KB - s.kb0) ? s.kb0 + static_cast<int>(left) : KB;
      u += s.kb1 - s.kb0;
      return true;
    }
    if (tile_it >= num_tiles) return false;
    s.tile = tile_it;
    s.kb0 = 0;
    s.kb1 = KB;
    tile_it += gridDim.x;
    return true;
  }
};

template <int BN_, int STAGES_, int TA_, int NACC_>
struct GemmCfg {
  static constexpr int BN = BN_, STAGES = STAGES_, TA = TA_, NACC = NACC_;
  static constexpr int kThreads = 384;
  static constexpr int kA8Bytes = BN * 128;
  static constexpr int kWBytes = kTileBytes;  // 8320
  static constexpr int kTmemCols = 512;
  static constexpr int kTmemA = NACC * BN;  // first column of the weight ring
  static_assert(NACC * BN + TA * 32 <= kTmemCols, "tensor memory budget");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
  static constexpr int kOffA8 = 0;
  static constexpr int kOffW = STAGES * kA8Bytes;
  static constexpr int kOffBar = (kOffW + STAGES * kWBytes + 15) / 16 * 16;
  static constexpr int kNumBars = 2 * STAGES + 2 * TA + 2 * NACC + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

enum : int {
  kErrProducer = 1,
  kErrMma = 2,
  kErrDequant = 3,
  kErrEpilogue = 4,
  kErrDrain = 5,
};

template <class C>
__global__ void __launch_bounds__(384, 1) w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                                                           const GemmArgs args) {
  constexpr int BN = C::BN, STAGES = C::STAGES, TA = C::TA, NACC = C::NACC;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA8 = smem + C::kOffA8;
  uint8_t* sW = smem + C::kOffW;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + TA;
  uint64_t* accfull = tempty + TA;
  uint64_t* accempty = accfull + NACC;
  uint64_t* done = accempty + NACC;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 2);
  volatile int* epi_fail = reinterpret_cast<volatile int*>(misc + 3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DevErr err{args.err};

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < TA; ++i) {
      mbar_init(&tfull[i], 4);
      mbar_init(&tempty[i], 1);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 4);
    }
    mbar_init(done, 1);
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 2) {
    tmem_alloc(&misc[0], C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_a);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  Sched sch;
  sch.init(args);
  Seg sg;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      int it = 0;
      bool ok = true;
      while (ok && sch.next(sg)) {
        const int m_tile = sg.tile % args.m_tiles, n_tile = sg.tile / args.m_tiles;
        const uint8_t* wsrc = args.tiles + static_cast<int64_t>(n_tile) * args.KB * kTileBytes;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, err, kErrProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::kA8Bytes + C::kWBytes);
          tma_load_2d(sA8 + s * C::kA8Bytes, &tmap_a, &full[s], kb * 128, m_tile * BN);
          bulk_load(sW + s * C::kWBytes, wsrc + static_cast<int64_t>(kb) * kTileBytes, C::kWBytes, &full[s],
                    pol_w);
        }
      }
      // Copies still in flight must land before the CTA may exit.
      const int first = it - STAGES > 0 ? it - STAGES : 0;
      for (int i = first; i < it; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, nullptr, err, kErrDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(128, BN);
      int it = 0, seg_i = 0;
      bool ok = true;
      while (ok && sch.next(sg)) {
        const int b = seg_i % NACC;
        const uint32_t bph = (seg_i / NACC) & 1;
        if (!mbar_wait(&accempty[b], bph ^ 1, abort_flag, err, kErrMma)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + b * BN;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
          const int s = it % STAGES, a = it % TA;
          const uint32_t ph = (it / STAGES) & 1, aph = (it / TA) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, err, kErrMma) ||
              !mbar_wait(&tfull[a], aph, abort_flag, err, kErrMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = tmem + C::kTmemA + a * 32;
          const uint32_t b_addr = smem_u32(sA8 + s * C::kA8Bytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_i8_ts(d_tmem, a_tmem + kk * 8, smem_desc_k128_sw128(b_addr + kk * 32), idesc,
                      (kb > sg.kb0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          mma_commit(&tempty[a]);
        }
        if (!ok) break;
        mma_commit(&accfull[b]);
        ++seg_i;
      }
      // every issued MMA must finish before TMEM is released
      mma_commit(done);
      mbar_wait(done, 0, nullptr, err, kErrDrain);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // --------------------------------------------------------- dequantizer
    const int qd = warp - 4;  // TMEM lane quarter
    const int r = qd * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    int it = 0;
    bool ok = true;
    while (ok && sch.next(sg)) {
      for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
        const int s = it % STAGES, a = it % TA;
        const uint32_t ph = (it / STAGES) & 1, aph = (it / TA) & 1;
        bool w_ok = mbar_wait(&full[s], ph, abort_flag, err, kErrDequant) &&
                    mbar_wait(&tempty[a], aph ^ 1, abort_flag, err, kErrDequant);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* wt = sW + s * C::kWBytes;
        const uint32_t meta = wt[kTileCodeBytes + r];
        const uint32_t zq = meta & 15u, s2 = (meta >> 4) + 1u;
        const uint32_t bias = (128u - zq * s2) * 0x01010101u;
        uint32_t out[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(wt + (c * kTileN + r) * 16);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            out[c * 8 + 2 * jj] = ((w[jj] & 0x0F0F0F0Fu) * s2 + bias) ^ 0x80808080u;
            out[c * 8 + 2 * jj + 1] = (((w[jj] >> 4) & 0x0F0F0F0Fu) * s2 + bias) ^ 0x80808080u;
          }
        }
        tmem_st_32(tmem + C::kTmemA + a * 32 + lane_base, out);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfull[a]);
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue
    const int qe = warp - 8;
    const uint32_t lane_base = static_cast<uint32_t>(qe * 32) << 16;
    const int64_t N = args.N;
    int seg_i = 0;
    bool ok = true;
    while (ok && sch.next(sg)) {
      const int b = seg_i % NACC;
      const uint32_t bph = (seg_i / NACC) & 1;
      // the four epilogue warps take one decision, so their named barriers
      // below are always reached by all of them
      ok = __all_sync(0xffffffffu, mbar_wait(&accfull[b], bph, abort_flag, err, kErrEpilogue));
      if (!ok && lane == 0) *epi_fail = 1;
      named_bar_sync(1, 128);
      ok = *epi_fail == 0;
      if (!ok) break;
      tc_fence_after();
      const int m_tile = sg.tile % args.m_tiles, n_tile = sg.tile / args.m_tiles;
      const int64_t n = static_cast<int64_t>(n_tile) * kTileN + qe * 32 + lane;
      const int m0 = m_tile * BN;
      const bool whole = (sg.kb0 == 0 && sg.kb1 == args.KB);
      const float s1f = __half2float(args.s1[n]);
      const uint32_t tb = tmem + b * BN + lane_base;
#pragma unroll 1
      for (int c = 0; c < BN; c += 16) {
        uint32_t v[16];
        tmem_ld_16(tb + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + c + j;
          if (m < args.M) {
            const int32_t acc = static_cast<int32_t>(v[j]);
            const int64_t o = static_cast<int64_t>(m) * N + n;
            if (!whole) {
              red_add_s32(args.ws_acc + o, acc);
            } else if (args.acc_out != nullptr) {
              args.acc_out[o] = acc;
            } else {
              const float scale = __fmul_rn(__half2float(args.sA[m]), s1f);
              args.Y[o] = __float2half_rn(__fmul_rn(__int2float_rn(acc), scale));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[b]);
      if (!whole) {
        // partial k-range: publish, take a ticket; the CTA that completes the
        // tile's k-blocks finishes it and restores the workspace to zero
        __threadfence();
        named_bar_sync(1, 128);
        if (qe == 0 && lane == 0) {
          const int add = sg.kb1 - sg.kb0;
          const int old = atomicAdd(args.ws_cnt + sg.tile, add);
          *last_flag = (old + add == args.KB) ? 1 : 0;
        }
        named_bar_sync(1, 128);
        if (*last_flag) {
          __threadfence();
          const int mend = min(m0 + BN, args.M);
          for (int m = m0; m < mend; ++m) {
            const int64_t o = static_cast<int64_t>(m) * N + n;
            const int32_t acc = __ldcg(args.ws_acc + o);
            __stcg(args.ws_acc + o, 0);
            if (args.acc_out != nullptr) {
              args.acc_out[o] = acc;
            } else {
              const float scale = __fmul_rn(__half2float(args.sA[m]), s1f);
              args.Y[o] = __float2half_rn(__fmul_rn(__int2float_rn(acc), scale));
            }
          }
          if (qe == 0 && lane == 0) args.ws_cnt[sg.tile] = 0;
        }
        named_bar_sync(1, 128);
      }
      ++seg_i;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace w4a8

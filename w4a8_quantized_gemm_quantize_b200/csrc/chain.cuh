// A chain of W4A8 GEMMs in one persistent launch, for the decode regime.
//
// Link j of the chain computes
//   (A8_j, sA_j, rowsum_j) = per-token int8 quantization of A_j (fp16)
//   Y_j = fp16_rn(float(sum_k A8_j W8_j) * (float(sA_j) * float(s1_j)))
// exactly as w4a8_quantize_act followed by w4a8_gemm, and link j reads A_j
// only after every output tile of link j - 1 is written, so A_j may be
// Y_{j-1} (a sequence of linear layers, each consuming the previous output).
//
// Why one launch: a decode GEMM streams a few to a few tens of MB of 4-bit
// weights, and launched one by one each GEMM pays a fixed chain of latencies
// at its start and end (CTA start-up, first weight bytes, the wait for the
// preceding kernel, the activation load queued behind the weight stream, the
// MMAs left after it, the split-k reduction and the epilogue), during which
// HBM idles. Here the weight stream never stops at a link boundary: the weight
// producer of every CTA runs through all links' weights in order, bounded only
// by its shared-memory ring, while the previous link finishes; the dependent
// part (quantize the activations, load them, the MMAs, the epilogue) is the
// only thing on the critical path between links. This follows the LiquidGEMM
// digest (arXiv 2509.01229, Method: weight loading, dequantization and MMA
// overlapped in one pipeline without software synchronization in the hot
// loop), taken across the GEMMs of a layer sequence.
//
// Work split: one CTA per SM. The output tiles (128 channels x up to 32
// tokens) of link j are cut into `split` k-ranges (1..4, as many as the SMs
// allow); segment g of the whole chain (links in order, then tiles, then
// ranks) runs on CTA g % grid, so the segments are dealt round robin across
// links. A tile cut into several k-ranges is reduced through the workspace:
// each rank stores its partial sums of the live token rows with plain
// stores, takes a ticket, and the last rank adds all of them (fixed order,
// so the result does not depend on timing) and writes Y.
//
// Ordering between CTAs: link j's token row m is quantized by CTA
// (seg0_j + m) % grid once `done[j - 1]` (output tiles finished) reaches the
// tile count of link j - 1 (for link 0: once the preceding kernel in the
// stream has completed); it then adds one to `ready[j]`, and the activation
// producers start loading link j's codes when `ready[j]` reaches M_j. Every
// such wait is bounded in time like every mbarrier wait of the library; the
// last CTA to leave resets the counters for the next launch.
#pragma once
#include "gemm.cuh"
#include "quantize_act.cuh"

namespace w4a8 {

constexpr int kChainMaxLinks = 16;
constexpr int kChainMaxM = 32;
constexpr int kChainMaxSplit = 4;  // k-ranges per output tile
constexpr int kErrChainWait = 9;  // W4A8_DEVERR_CHAIN_WAIT

struct ChainLink {
  const uint8_t* tiles;  // packed weight tiles (blob + header)
  const __half* s1;      // per-output-channel scales (inside the blob)
  const __half* A;       // fp16 activations [M, K]
  int8_t* A8;            // their int8 codes [M, K] (written by the chain)
  __half* sA;            // per-token scales [M] (written by the chain)
  int32_t* rowsum;       // per-token code sums [M] (written by the chain)
  __half* Y;             // output [M, N]
  int32_t* part;         // split > 1: partial sums [num_tiles][split][M][128]
  int32_t* ticket;       // split > 1: [num_tiles], zero between launches
  int M, N, KB;
  int num_tiles;         // N / 128
  int split;             // k-ranges (CTAs) per output tile
  int seg0;              // index of the link's first segment in the chain
};

struct ChainArgs {
  ChainLink link[kChainMaxLinks];
  int n_links;
  int32_t* done;   // [n_links] finished output tiles, zero between launches
  int32_t* ready;  // [n_links] quantized token rows, zero between launches
  int32_t* exits;  // CTAs that finished; the last one zeroes done, ready and exits
  int* err;        // device error word
};

// TMA descriptors of the links' int8 codes (box 128 bytes x 32 rows,
// 128-byte swizzle; rows past M read as zeros).
struct ChainMaps {
  CUtensorMap m[kChainMaxLinks];
};

struct ChainSeg {
  int link, tile, rank, kb0, kb1;
};

// Replays this CTA's segments in chain order (every role walks the same list).
struct ChainSched {
  int j, s;
  __device__ __forceinline__ static int first(const ChainArgs& a, int jj) {
    const int G = static_cast<int>(gridDim.x);
    const int off = (static_cast<int>(blockIdx.x) - a.link[jj].seg0) % G;
    return off < 0 ? off + G : off;
  }
  __device__ __forceinline__ void init(const ChainArgs& a) {
    j = 0;
    s = a.n_links > 0 ? first(a, 0) : 0;
  }
  __device__ __forceinline__ bool next(const ChainArgs& a, ChainSeg& g) {
    while (j < a.n_links) {
      const ChainLink& L = a.link[j];
      if (s < L.num_tiles * L.split) {
        g.link = j;
        g.tile = s / L.split;
        g.rank = s - g.tile * L.split;
        g.kb0 = L.KB * g.rank / L.split;
        g.kb1 = L.KB * (g.rank + 1) / L.split;
        s += static_cast<int>(gridDim.x);
        return true;
      }
      if (++j < a.n_links) s = first(a, j);
    }
    return false;
  }
};

// Waits until *p >= target (p written by other CTAs: acquire loads), with the
// same time bound as every mbarrier wait. Returns false on abort or expiry.
__device__ __forceinline__ bool chain_wait_counter(const int32_t* p, int target, volatile int* abort_flag,
                                                   DevErr err) {
  if (ld_acquire_gpu(p) >= target) return true;
  uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (ld_acquire_gpu(p) >= target) return true;
    if ((it & 15u) == 0) {
      if (abort_flag != nullptr && *abort_flag) return false;
      const uint64_t now = global_timer_ns();
      if (now < t0 || (err.armed != nullptr && *err.armed == 0)) {
        t0 = now;
      } else if (now - t0 > kWaitLimitNs) {
        if (abort_flag != nullptr) *abort_flag = 1;
        atomicCAS(err.word, 0, kErrChainWait);
        return false;
      }
    }
  }
}

// Quantizes token row m of link L with the 128 threads of the epilogue group
// (thread t, named barrier 1, 4 + 4 words of shared memory): the arithmetic
// of quantize_act_kernel (amax, sA = fp16_rn(amax / 127), codes
// clamp(rint(A / float(sA)), -127, 127) with IEEE divides, rowsum). Rows of
// up to 128 x kQuantVecs 16-byte vectors (K <= 14336) are loaded once, every
// load issued before the first is used, and coded from registers; longer rows
// take two passes in batches of 8 vectors per thread.
constexpr int kQuantVecs = 14;

__device__ __forceinline__ float amax_of(const uint4& v, float a) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __half22float2(h[j]);
    a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
  }
  return a;
}

// The 8 codes of one 16-byte vector (as 8 bytes) and their sum.
__device__ __forceinline__ uint2 codes_of(const uint4& v, float sf, int& local) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint32_t w[2] = {0u, 0u};
  if (sf != 0.0f) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(h[j]);
      const int q0 = quant_code<127>(f.x, sf), q1 = quant_code<127>(f.y, sf);
      local += q0 + q1;
      w[j >> 1] |= ((static_cast<uint32_t>(q0) & 0xFFu) | ((static_cast<uint32_t>(q1) & 0xFFu) << 8))
                   << ((j & 1) * 16);
    }
  }
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ void chain_quantize_row(const ChainLink& L, int m, int t, float* fred, int* ired) {
  const int64_t K = static_cast<int64_t>(L.KB) * kTileK;
  const int nvec = static_cast<int>(K >> 3);
  const uint4* row = reinterpret_cast<const uint4*>(L.A + m * K);
  uint2* out = reinterpret_cast<uint2*>(L.A8 + m * K);
  const int warp = t >> 5, lane = t & 31;
  float amax = 0.0f;
  int local = 0;
  uint4 v[kQuantVecs];
  const bool one_pass = nvec <= 128 * kQuantVecs;
  if (one_pass) {
#pragma unroll
    for (int i = 0; i < kQuantVecs; ++i) {
      const int idx = t + 128 * i;
      v[i] = __ldcg(row + (idx < nvec ? idx : nvec - 1));  // in-bounds address; the guard below selects
    }
#pragma unroll
    for (int i = 0; i < kQuantVecs; ++i)
      if (t + 128 * i < nvec) amax = amax_of(v[i], amax);
  } else {
    for (int base = 0; base < nvec; base += 128 * 8) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int idx = base + t + 128 * i;
        v[i] = __ldcg(row + (idx < nvec ? idx : nvec - 1));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (base + t + 128 * i < nvec) amax = amax_of(v[i], amax);
    }
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) fred[warp] = amax;
  named_bar_sync(1, 128);
  amax = fmaxf(fmaxf(fred[0], fred[1]), fmaxf(fred[2], fred[3]));
  const __half s_h = __float2half_rn(__fdiv_rn(amax, 127.0f));
  const float sf = __half2float(s_h);
  if (one_pass) {
#pragma unroll
    for (int i = 0; i < kQuantVecs; ++i) {
      const int idx = t + 128 * i;
      if (idx < nvec) out[idx] = codes_of(v[i], sf, local);  // idx < nvec: inside row m of [M, K]
    }
  } else {
    for (int base = 0; base < nvec; base += 128 * 8) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int idx = base + t + 128 * i;
        v[i] = __ldcg(row + (idx < nvec ? idx : nvec - 1));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int idx = base + t + 128 * i;
        if (idx < nvec) out[idx] = codes_of(v[i], sf, local);
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if (lane == 0) ired[warp] = local;
  named_bar_sync(1, 128);
  if (t == 0) {
    L.rowsum[m] = ired[0] + ired[1] + ired[2] + ired[3];
    L.sA[m] = s_h;
  }
  // the codes are read by TMA (async proxy) in other CTAs
  fence_proxy_async_global();
  named_bar_sync(1, 128);
}

// Writes 16 token rows x this warp's 32 output channels of link L
// (16-byte stores through the warp's shared-memory stage, rows >= M skipped).
__device__ __forceinline__ void chain_store_rows16(const ChainLink& L, __half* stage, const __half (&h)[16], int m_start,
                                                   int64_t n_base, int lane, int* err) {
#pragma unroll
  for (int j = 0; j < 16; ++j) stage[j * 32 + lane] = h[j];
  __syncwarp();
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int r = pass * 8 + (lane >> 2), q = lane & 3;
    const uint4 v = *reinterpret_cast<const uint4*>(stage + r * 32 + q * 8);
    const int m = m_start + r;
    if (m < L.M && in_bounds(n_base >= 0 && n_base + q * 8 + 8 <= L.N, err))
      *reinterpret_cast<uint4*>(L.Y + static_cast<int64_t>(m) * L.N + n_base + q * 8) = v;
  }
  __syncwarp();
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1) w4a8_chain_kernel(const __grid_constant__ ChainMaps maps,
                                                                     const __grid_constant__ ChainArgs args) {
  constexpr int BN = C::BN, KS = C::KS, NS = C::NS, NT = C::NT, DQ = C::DQ, NACC = C::NACC, NMMA = C::NMMA;
  static_assert(BN == kChainMaxM && !C::kLut, "the chain runs the 32-token int8 configuration");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA8 = smem + C::kOffA8;
  uint8_t* sW = smem + C::kOffW;
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* wempty = wfull + NS;
  uint64_t* afull = wempty + NS;
  uint64_t* aempty = afull + NS;
  uint64_t* tfull = aempty + NS;
  uint64_t* tempty = tfull + NT;
  uint64_t* accfull = tempty + NT;
  uint64_t* accempty = accfull + NACC;
  uint64_t* mma_done = accempty + NACC;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 2);
  volatile int* epi_fail = reinterpret_cast<volatile int*>(misc + 3);
  volatile int* dep_done = reinterpret_cast<volatile int*>(misc + 4);
  float* fred = reinterpret_cast<float*>(misc + 8);  // 4 words
  int* ired = reinterpret_cast<int*>(misc + 12);     // 4 words

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DevErr err{args.err, dep_done};

  if (warp == 1) {
    // weight starter: the first chunks' copies go out before the set-up
    if (lane == 0) {
      for (int i = 0; i < NS; ++i) {
        mbar_init(&wfull[i], 1);
        mbar_init(&wempty[i], 4);
      }
      fence_barrier_init();
      fence_proxy_async_smem();
      const uint64_t pol_w = l2_policy_evict_first();
      ChainSched s0;
      s0.init(args);
      ChainSeg g0;
      int c = 0;
      while (c < C::kStartChunks && s0.next(args, g0)) {
        const ChainLink& L = args.link[g0.link];
        const uint8_t* wsrc = L.tiles + static_cast<int64_t>(g0.tile) * L.KB * C::kTileB;
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
    }
    for (int i = 0; i < NT; ++i) {
      mbar_init(&tfull[i], 4);
      mbar_init(&tempty[i], 1);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&accfull[i], NMMA);
      mbar_init(&accempty[i], 4);
    }
    mbar_init(mma_done, NMMA);
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;
    misc[4] = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(&misc[0], C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 3 && lane < args.n_links) prefetch_tensormap(&maps.m[lane]);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  ChainSched sch;
  sch.init(args);
  ChainSeg sg;

  if (warp == 0) {
    // ----------------------------------------------------- weight producer
    // Runs through every link's weights without waiting for any activation:
    // only the ring's free slots pace it.
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      int c = 0;
      bool ok = true;
      while (ok && sch.next(args, sg)) {
        const ChainLink& L = args.link[sg.link];
        const uint8_t* wsrc = L.tiles + static_cast<int64_t>(sg.tile) * L.KB * C::kTileB;
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
      grid_launch_dependents();  // every weight byte of this CTA is requested
      const int first = c - NS > 0 ? c - NS : 0;
      for (int i = first; i < c; ++i) mbar_wait(&wfull[i % NS], (i / NS) & 1, nullptr, err, kErrDrain);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------- activation producer
    if (lane == 0) {
      grid_dependency_wait();
      *dep_done = 1;
      int c = 0, cur = -1;
      bool ok = true;
      while (ok && sch.next(args, sg)) {
        const ChainLink& L = args.link[sg.link];
        if (sg.link != cur) {
          // the link's codes are complete once all its token rows are counted
          cur = sg.link;
          if (!chain_wait_counter(&args.ready[cur], L.M, abort_flag, err)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();  // TMA reads after the acquire of the codes other CTAs wrote
        }
        for (int kb = sg.kb0; kb < sg.kb1; kb += KS, ++c) {
          const int cnt = min(KS, sg.kb1 - kb);
          const int a = c % NS;
          if (!mbar_wait(&aempty[a], ((c / NS) & 1) ^ 1, abort_flag, err, kErrProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&afull[a], cnt * C::kA8Bytes);
          for (int j = 0; j < cnt; ++j)
            tma_load_2d(sA8 + a * C::kASlot + j * C::kA8Bytes, &maps.m[sg.link], &afull[a], (kb + j) * kTileK, 0);
        }
      }
      const int first = c - NS > 0 ? c - NS : 0;
      for (int i = first; i < c; ++i) mbar_wait(&afull[i % NS], (i / NS) & 1, nullptr, err, kErrDrain);
    }
    __syncwarp();
  } else if (warp >= 1 && warp < 1 + NMMA) {
    // ----------------------------------------------------------- MMA issuers
    if (lane == 0) {
      const int mi = warp - 1;
      constexpr uint32_t idesc = idesc_i8(128, BN);
      int c = 0, seg_i = 0;
      bool ok = true;
      while (ok && sch.next(args, sg)) {
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
            for (int kk = 0; kk < C::kMmaPerKb; ++kk)
              mma_i8_ts(d_tmem, a_tmem + j * C::kKbCols + kk * 8,
                        smem_desc_k128_sw128(b_addr + j * C::kA8Bytes + kk * 32), idesc, 1u);
          }
          mma_commit(&aempty[a]);
          mma_commit(&tempty[t]);
        }
        if (!ok) break;
        mma_commit(&accfull[b]);
        ++seg_i;
      }
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, err, kErrDrain);
    }
    __syncwarp();
  } else if (warp >= C::kDqWarp0 && warp < C::kDqWarp0 + 4 * DQ) {
    // --------------------------------------------------------- dequantizers
    const int g = (warp - C::kDqWarp0) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int c = 0, prev_t = -1;
    bool ok = true;
    while (ok && sch.next(args, sg)) {
      for (int kb = sg.kb0; kb < sg.kb1; kb += KS, ++c) {
        if (c % DQ != g) continue;
        const int cnt = min(KS, sg.kb1 - kb);
        const int w = c % NS, t = c % NT;
        if (!__all_sync(0xffffffffu, mbar_wait(&tempty[t], ((c / NT) & 1) ^ 1, abort_flag, err, kErrDequant) &&
                                         mbar_wait(&wfull[w], (c / NS) & 1, abort_flag, err, kErrDequant))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < cnt; ++j) {
          uint32_t out[32];
          dequant_tile_regs(sW + w * C::kWSlot + j * C::kTileB, r, out);
          if (C::kPipelinedStores && j == 0 && prev_t >= 0) {
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tfull[prev_t]);
          }
          tmem_st_32(tmem + C::kTmemA + t * C::kTSlotCols + j * C::kKbCols + lane_base, out);
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
    // -------------------------------------- quantizers of rows and epilogue
    grid_dependency_wait();  // link 0's activations may come from the preceding kernel
    const int quarter = warp & 3;
    const int t = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int32_t* rs_stage = reinterpret_cast<int32_t*>(smem + C::kOffRows);
    float* sa_stage = reinterpret_cast<float*>(smem + C::kOffRows + 512);
    __half* ystage = reinterpret_cast<__half*>(smem + C::kOffYStage + quarter * 1024);
    for (int b = 0; b < NACC; ++b)
      for (int cc = 0; cc < BN; cc += 16) tmem_zero_16(tmem + b * BN + cc + lane_base);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
      for (int b = 0; b < NACC; ++b) mbar_arrive(&accempty[b]);
    const int G = static_cast<int>(gridDim.x);
    int seg_i = 0;
    bool ok = true;
    for (int j = 0; j < args.n_links && ok; ++j) {
      const ChainLink& L = args.link[j];
      // ---- this CTA's token rows of link j (rows m with (seg0 + m) % G == this CTA)
      for (int m = ChainSched::first(args, j); m < L.M; m += G) {
        if (j > 0) {
          bool w = true;
          if (t == 0) {
            w = chain_wait_counter(&args.done[j - 1], args.link[j - 1].num_tiles, abort_flag, err);
            if (!w) *epi_fail = 1;
          }
          named_bar_sync(1, 128);
          if (*epi_fail) {
            ok = false;
            break;
          }
        }
        chain_quantize_row(L, m, t, fred, ired);
        if (t == 0) {
          fence_acq_rel_gpu();
          atomicAdd(&args.ready[j], 1);
        }
      }
      if (!ok) break;
      // ---- epilogues of this CTA's segments of link j
      const int nseg = L.num_tiles * L.split;
      for (int s = ChainSched::first(args, j); s < nseg; s += G) {
        const int tile = s / L.split, rank = s - tile * L.split;
        const int b = seg_i % NACC;
        // the link's per-token operands (written by the quantizing CTAs)
        if (t < BN) {
          float sa = 0.0f;
          int32_t rsum = 0;
          if (t < L.M && chain_wait_counter(&args.ready[j], L.M, abort_flag, err)) {
            sa = __half2float(L.sA[t]);
            rsum = L.rowsum[t];
          }
          sa_stage[t] = sa;
          rs_stage[t] = rsum;
        }
        bool w = mbar_wait(&accfull[b], (seg_i / NACC) & 1, abort_flag, err, kErrEpilogue);
        w = __all_sync(0xffffffffu, w);
        if (!w && lane == 0) *epi_fail = 1;
        named_bar_sync(1, 128);
        if (*epi_fail) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[BN];
#pragma unroll
        for (int cc = 0; cc < BN; cc += 16) {
          uint32_t u[16];
          tmem_ld_16_wait(tmem + b * BN + cc + lane_base, u);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) v[cc + jj] = u[jj];
          tmem_zero_16(tmem + b * BN + cc + lane_base);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[b]);
        ++seg_i;
        const int64_t n = static_cast<int64_t>(tile) * kTileN + t;
        bool finish = true;
        if (L.split > 1) {
          // partial sums of the live rows, then the ticket: the last rank finishes the tile
          int32_t* mine = L.part + (static_cast<int64_t>(tile) * L.split + rank) * L.M * kTileN + t;
          const bool part_ok = in_bounds(tile < L.num_tiles && rank < L.split && L.part != nullptr, args.err);
#pragma unroll
          for (int mm = 0; mm < BN; ++mm)
            if (mm < L.M && part_ok) mine[mm * kTileN] = static_cast<int32_t>(v[mm]);
          named_bar_sync(1, 128);
          if (t == 0) {
            fence_acq_rel_gpu();
            const int old = atomicAdd(L.ticket + tile, 1);
            fence_acq_rel_gpu();
            *last_flag = (old == L.split - 1) ? 1 : 0;
          }
          named_bar_sync(1, 128);
          finish = *last_flag != 0;
        }
        if (finish) {
          const float s1f = __half2float(L.s1[n]);
#pragma unroll
          for (int cc = 0; cc < BN; cc += 16) {
            uint32_t x[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) x[jj] = v[cc + jj];
            if (L.split > 1) {
              // the sum of every rank's partial sums (this CTA's included, in
              // rank order), 8 rows at a time with all their loads issued
              // before the adds
              const bool part_ok = in_bounds(tile < L.num_tiles && L.part != nullptr, args.err);
              int32_t* base = L.part + static_cast<int64_t>(tile) * L.split * L.M * kTileN + t;
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                int32_t p[kChainMaxSplit][8];
#pragma unroll
                for (int rr = 0; rr < kChainMaxSplit; ++rr)
#pragma unroll
                  for (int jj = 0; jj < 8; ++jj) {
                    const int mm = cc + 8 * half + jj;
                    p[rr][jj] = (rr < L.split && mm < L.M && part_ok)
                                    ? __ldcg(base + (static_cast<int64_t>(rr) * L.M + mm) * kTileN)
                                    : 0;
                  }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                  uint32_t sum = 0u;
#pragma unroll
                  for (int rr = 0; rr < kChainMaxSplit; ++rr) sum += static_cast<uint32_t>(p[rr][jj]);
                  x[8 * half + jj] = sum;
                }
#pragma unroll
                for (int rr = 0; rr < kChainMaxSplit; ++rr)
#pragma unroll
                  for (int jj = 0; jj < 8; ++jj) {
                    const int mm = cc + 8 * half + jj;
                    if (rr < L.split && mm < L.M && part_ok)
                      __stcg(base + (static_cast<int64_t>(rr) * L.M + mm) * kTileN, 0);  // left zero-filled
                  }
              }
            }
            __half h[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              h[jj] = output_half(x[jj], rs_stage[cc + jj], sa_stage[cc + jj], s1f);
            chain_store_rows16(L, ystage, h, cc, n - lane, lane, args.err);
          }
          if (L.split > 1 && t == 0) L.ticket[tile] = 0;  // ready for the next launch
          named_bar_sync(1, 128);
          if (t == 0) {
            fence_acq_rel_gpu();
            atomicAdd(&args.done[j], 1);  // one more output tile of link j is complete
          }
        }
        named_bar_sync(1, 128);  // the stages are reused by the next segment
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  if (threadIdx.x == 0) {
    // the last CTA to leave resets the counters (every other CTA is past all
    // its waits on them)
    fence_acq_rel_gpu();
    if (atomicAdd(args.exits, 1) == static_cast<int>(gridDim.x) - 1) {
      fence_acq_rel_gpu();
      for (int j = 0; j < args.n_links; ++j) {
        args.done[j] = 0;
        args.ready[j] = 0;
      }
      fence_acq_rel_gpu();
      *args.exits = 0;
    }
  }
}

}  // namespace w4a8

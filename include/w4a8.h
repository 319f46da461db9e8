/*
 * w4a8.h — C ABI of the B200 (sm_100a) W4A8 quantized GEMM library.
 *
 * The operation is the W4A8 GEMM of QServe/QoQ: 4-bit weights, 8-bit
 * activations, with a progressive (two-level) weight quantization that keeps
 * dequantization inside the GEMM cheap ("QServe/QoQ" abstract, quoted in the
 * lmdeploy issue "[Feature] Support W4A8KV4 Quantization(QServe/QoQ)",
 * Motivation; "LiquidGEMM: Hardware-Efficient W4A8 GEMM Kernel for
 * High-Performance LLM Serving", Method):
 *
 *   W8[n,k] = (q[n,k] - z[n,g]) * s2[n,g]        g = k / 128, exact int8
 *   acc[m,n] = sum_k A8[m,k] * W8[n,k]            int32
 *   Y[m,n]  = fp16_rn(float(acc) * (float(sA[m]) * float(s1[n])))
 *
 * with q, z in [0, 15] (uint4), s2 in [1, 8], s1 a per-output-channel fp16
 * scale and (A8, sA) the per-token symmetric int8 quantization of the fp16
 * activations.
 *
 * Conventions for every call:
 *  - All data pointers are DEVICE pointers, allocated and owned by the
 *    caller; the library allocates, frees and synchronizes nothing (except
 *    w4a8_get_device_error, which synchronizes the given stream).
 *  - Work is enqueued on `stream` (NULL = the legacy default stream) and is
 *    asynchronous; a returned W4A8_OK means "validated and launched".
 *  - Arguments are validated on the host before any launch; on error nothing
 *    is launched. A launch failure returns W4A8_ERR_CUDA after reading (and
 *    thereby clearing) the CUDA runtime's last error.
 *  - Data pointers must be 16-byte aligned unless stated otherwise.
 *  - Matrices are row-major and dense (leading dimension = row length).
 *  - The activation quantizers and the GEMM launch as programmatic
 *    dependents of the preceding kernel in the stream: they may start while
 *    it still runs and wait for it to complete before they read or write
 *    anything of it, with one exception: the GEMM starts reading the packed
 *    weight blob at once. The blob must therefore be complete before the
 *    kernel just ahead of the GEMM in the stream starts (w4a8_pack_weights
 *    and any ordinary kernel or copy satisfy this; only a kernel that itself
 *    releases its dependents early could break it, by writing the blob).
 */
#ifndef W4A8_H_
#define W4A8_H_

#include <stddef.h>
#include <stdint.h>

#if defined(W4A8_BUILD)
#define W4A8_API __attribute__((visibility("default")))
#else
#define W4A8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* w4a8_stream_t;

typedef enum {
  W4A8_OK = 0,
  W4A8_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad option */
  W4A8_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside the documented limits */
  W4A8_ERR_MISALIGNED = 3,        /* pointer not aligned as required */
  W4A8_ERR_WORKSPACE = 4,         /* workspace missing or too small */
  W4A8_ERR_CUDA = 5,              /* CUDA runtime / launch error */
  W4A8_ERR_DEVICE = 6             /* a kernel gave up a bounded wait (see below) */
} w4a8_status_t;

/* Device error word values (w4a8_get_device_error). */
#define W4A8_DEVERR_NONE 0
#define W4A8_DEVERR_PRODUCER_WAIT 1
#define W4A8_DEVERR_MMA_WAIT 2
#define W4A8_DEVERR_DEQUANT_WAIT 3
#define W4A8_DEVERR_EPILOGUE_WAIT 4
#define W4A8_DEVERR_DRAIN_WAIT 5
#define W4A8_DEVERR_SELFTEST_WAIT 6
#define W4A8_DEVERR_KV_RANGE 7 /* a KV-cache length or position outside [0, Lmax] (clamped or skipped) */
#define W4A8_DEVERR_PACK_RANGE 8 /* a packer met a code, zero point or scale outside its documented range */
#define W4A8_DEVERR_CHAIN_WAIT 9 /* w4a8_chain: a wait on another CTA's progress gave up */
#define W4A8_DEVERR_BOUNDS 10     /* debug builds (W4A8_DEBUG) only: an access outside its buffer was skipped */
#define W4A8_DEVERR_KV_WAIT 11    /* w4kv_attention_decode: a chunk's cache copies did not land in time */

/* Human-readable name of a status code (static string, never NULL). */
W4A8_API const char* w4a8_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
W4A8_API int w4a8_version(void);

/*
 * Per-token symmetric int8 quantization of activations (the 8-bit activation
 * side of W4A8; per-token dynamic scaling as in the "PrefixQuant" page, Key
 * Findings). For each row m:
 *   amax = max_k |A[m,k]|
 *   sA[m] = fp16_rn(amax / 127)                       (IEEE fp32 divide)
 *   A8[m,k] = clamp(rint(A[m,k] / float(sA[m])), -127, 127)
 *                                     (IEEE fp32 divide, ties to even)
 *   sA[m] == 0 gives A8[m,:] = 0;  rowsum[m] = sum_k A8[m,k].
 * A: fp16 [M, K]. A8: int8 [M, K]. sA: fp16 [M] (2-byte aligned).
 * rowsum: int32 [M] (4-byte aligned) or NULL.
 * Limits: M >= 0 (M == 0 is a no-op), 0 < K <= 65536, K % 8 == 0.
 * Non-finite inputs are a precondition violation (codes unspecified).
 */
W4A8_API w4a8_status_t w4a8_quantize_act(const void* A, int64_t M, int64_t K, int8_t* A8, void* sA, int32_t* rowsum,
                                w4a8_stream_t stream);

/*
 * Per-tensor static symmetric int8 quantization: one fp16 scale for the
 * whole activation tensor, calibrated offline ("PrefixQuant: Static
 * Quantization Beats Dynamic through Prefixed Outliers in LLMs",
 * Methodology and Key Findings: per-tensor static quantization once the
 * outlier tokens are prefixed). No amax pass:
 *   A8[m,k] = clamp(rint(A[m,k] / float(s)), -127, 127)
 *                                     (IEEE fp32 divide, ties to even)
 *   s == 0 gives all-zero codes; rowsum[m] = sum_k A8[m,k]; sA[m] = s, so
 *   the result feeds w4a8_gemm unchanged.
 * s: device pointer to ONE fp16 value (read on the device, so a captured
 * graph picks up a changed scale). Other arguments and limits as for
 * w4a8_quantize_act.
 */
W4A8_API w4a8_status_t w4a8_quantize_act_static(const void* A, int64_t M, int64_t K, const void* s, int8_t* A8,
                                                void* sA, int32_t* rowsum, w4a8_stream_t stream);

/*
 * Offline two-level weight quantization (the "progressive quantization" of
 * the QServe/QoQ abstract), fp32 W [N, K] -> (q, z, s2, s1):
 *   level 1 (row n): r_g = max(max W_g, 0) - min(min W_g, 0) over each
 *     group g of 128; s1[n] = fp16_rn(max_g r_g / 120), 1 if that is 0;
 *     t = W / float(s1[n]).
 *   level 2 (group): lo = min(min t, 0), hi = max(max t, 0);
 *     s2 = clamp(ceil((hi - lo) / 15), 1, 8);  z = clamp(rint(-lo / s2), 0, 15);
 *     q = clamp(rint(t / s2) + z, 0, 15).          (IEEE fp32 divides)
 * so that (q - z) * s2 lies in [-120, 120].
 * q: uint8 [N, K] one code per byte. z, s2: uint8 [N, K/128] (no alignment
 * requirement). s1: fp16 [N] (2-byte aligned).
 * Limits: group == 128, K % 128 == 0, 0 < K <= 65536, N >= 0.
 */
W4A8_API w4a8_status_t w4a8_quantize_weights(const float* W, int64_t N, int64_t K, int32_t group, uint8_t* q, uint8_t* z,
                                    uint8_t* s2, void* s1, w4a8_stream_t stream);

/* Size in bytes of the packed blob for an N x K weight (0 if unsupported). */
W4A8_API size_t w4a8_packed_bytes(int64_t N, int64_t K, int32_t group);

/*
 * Offline reordering of (q, z, s2, s1) into the GEMM's packed blob
 * (compute-aware weight reordering, "QServe/QoQ" abstract; offline
 * interleaving, "QUICK" abstract). Layout, little-endian:
 *   header, 64 bytes: u32 magic "W4A8", u32 version 1, i64 N, i64 K,
 *     i32 group, u32 tile bytes (8320), u64 byte offset of s1, zeros.
 *   tiles: (N/128) x (K/128) tiles of 8320 bytes; tile (nt, kt) at
 *     64 + (nt * K/128 + kt) * 8320 holds 8192 code bytes then 128 meta bytes.
 *     Row r (n = 128 nt + r) keeps the codes of in-tile k = 8j .. 8j+7 in
 *     32-bit word j, byte b holding k = 8j+b (low nibble) and k = 8j+4+b
 *     (high nibble); word j of row r is word ((j/4)*128 + r)*4 + j%4 of the
 *     tile. Meta byte r = z | ((s2 - 1) << 4) of group kt.
 *   s1: N fp16 values, zero padded to a multiple of 16 bytes.
 * q/z/s2/s1 as produced by w4a8_quantize_weights (q and s1 16-byte aligned):
 * q and z in [0, 15], s2 in [1, 8]. A value outside its range is reported as
 * W4A8_DEVERR_PACK_RANGE in the device error word (its field keeps only the
 * low bits, so the blob is then wrong).
 * packed: packed_bytes >= w4a8_packed_bytes(N, K, group).
 * Limits: group == 128, N % 128 == 0, K % 128 == 0, 0 < K <= 65536.
 */
W4A8_API w4a8_status_t w4a8_pack_weights(const uint8_t* q, const uint8_t* z, const uint8_t* s2, const void* s1, int64_t N,
                                int64_t K, int32_t group, void* packed, size_t packed_bytes, w4a8_stream_t stream);

/*
 * Workspace for w4a8_gemm / w4a8_gemm_debug_acc / w4a8_gemm_ex: int32
 * partial sums and per-tile tickets used when one output tile's k-range is
 * split across CTAs that are not in one cluster (the decode regime with
 * more tiles than fit one cluster each; the cluster split needs none). The caller zero-fills it ONCE before
 * first use; every call that completes without a device error leaves it
 * zero-filled again. Calls that share a workspace must not overlap in time.
 * A workspace of the returned size serves every M' <= M, N' <= N.
 */
W4A8_API size_t w4a8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * Y = fp16(sA[m] * s1[n] * sum_k A8[m,k] * W8[n,k]), W8 decoded from the
 * packed blob in registers (see the top of this file).
 * A8: int8 [M, K] (from w4a8_quantize_act). sA: fp16 [M] (2-byte aligned).
 * rowsum: int32 [M] (4-byte aligned), rowsum[m] = sum_k A8[m,k] as written
 *   by w4a8_quantize_act. The kernel multiplies the weights in the biased
 *   unsigned form W8 + 128 (no sign fix-up while dequantizing) and subtracts
 *   128 * rowsum[m] exactly; a rowsum that does not match A8 gives wrong
 *   results.
 * packed: the blob of w4a8_pack_weights for exactly this N and K.
 * Y: fp16 [M, N]. workspace: see w4a8_gemm_workspace_bytes; with too small a
 * workspace (including NULL / 0) the call uses a schedule that needs none.
 * Limits: M >= 0 (M == 0 is a no-op), N % 128 == 0, K % 128 == 0,
 * 0 < K <= 65536, M * N < 2^62.
 */
W4A8_API w4a8_status_t w4a8_gemm(const int8_t* A8, const void* sA, const int32_t* rowsum, const void* packed,
                                 int64_t M, int64_t N, int64_t K, void* Y, void* workspace, size_t workspace_bytes,
                                 w4a8_stream_t stream);

/*
 * Debug entry point: the same GEMM, writing the int32 accumulators
 * acc[m,n] = sum_k A8[m,k] * W8[n,k] to `acc` [M, N] instead of Y
 * (rowsum as for w4a8_gemm).
 */
W4A8_API w4a8_status_t w4a8_gemm_debug_acc(const int8_t* A8, const int32_t* rowsum, const void* packed, int64_t M,
                                           int64_t N, int64_t K, int32_t* acc, void* workspace,
                                           size_t workspace_bytes, w4a8_stream_t stream);

/* Scheduling overrides for tests and tuning (zero = automatic). */
typedef struct {
  int32_t schedule;  /* 0 auto, 1 whole tiles per CTA, 2 split k-ranges (needs workspace),
                        3 cluster split (block_m <= 32: each tile's k-range split over the
                        2..4 CTAs of one thread-block cluster, reduced on chip; needs no
                        workspace; W4A8_ERR_UNSUPPORTED_SHAPE if the tiles do not fit
                        one cluster each) */
  int32_t block_m;   /* tokens per tile: 0 auto, or 16, 32, 64, 128 */
  int32_t max_ctas;  /* 0 auto (one CTA per SM), else an upper bound on the grid */
  int32_t reserved;  /* must be 0 */
} w4a8_gemm_opts_t;

/*
 * w4a8_gemm with overrides. Exactly one of Y (fp16 output) and acc (int32
 * accumulators) must be non-NULL; sA may be NULL when acc is given.
 * opts may be NULL (= all automatic).
 */
W4A8_API w4a8_status_t w4a8_gemm_ex(const int8_t* A8, const void* sA, const int32_t* rowsum, const void* packed,
                                    int64_t M, int64_t N, int64_t K, void* Y, int32_t* acc, void* workspace,
                                    size_t workspace_bytes, const w4a8_gemm_opts_t* opts, w4a8_stream_t stream);

/*
 * GEMM chain for the decode regime: a sequence of up to 16 W4A8 GEMMs ("links")
 * in ONE persistent launch. Link j computes exactly what
 *   w4a8_quantize_act(A_j) -> (A8_j, sA_j, rowsum_j);  w4a8_gemm(...) -> Y_j
 * computes (bit for bit), in order: link j's activations A_j are read only
 * after every element of Y_{j-1} is written (link 0's after the preceding
 * kernel in the stream has completed), so A_j may be Y_{j-1} (K_j == N_{j-1})
 * or anything computed before the call. The weight stream of all links runs
 * ahead without waiting on any activation: in a per-GEMM launch sequence every
 * launch pays a chain of start-up and tail latencies during which HBM idles,
 * here only the dependent part (quantize, load the codes, the remaining MMAs,
 * the epilogue) sits between links ("LiquidGEMM: Hardware-Efficient W4A8 GEMM
 * Kernel for High-Performance LLM Serving", Method: weight loading,
 * dequantization and MMA overlapped in one pipeline).
 *
 * links: HOST array of n_links link descriptors (1 <= n_links <= 16), read
 * during the call. Per link: A fp16 [M, K] (16-byte aligned); packed the blob
 * of w4a8_pack_weights for N x K; A8 int8 [M, K] (16-byte aligned), sA fp16
 * [M] (2-byte aligned), rowsum int32 [M] (4-byte aligned): written with the
 * link's quantized activations (links may share these three buffers); Y fp16
 * [M, N] (16-byte aligned). Limits per link: 1 <= M <= 32, N % 128 == 0,
 * K % 128 == 0, 0 < K <= 65536.
 * workspace: 256-byte aligned, at least w4a8_chain_workspace_bytes(links,
 * n_links) bytes (it depends on the shapes and the device's SM count),
 * zero-filled by the caller once; every call that completes without a device
 * error leaves it zero-filled again. Calls sharing a workspace must not
 * overlap on the GPU. The launch uses one CTA per SM and needs all of them
 * resident at once (its CTAs wait on each other's progress; every such wait
 * is bounded and reports W4A8_DEVERR_CHAIN_WAIT if it gives up, after which
 * the workspace must be zero-filled again).
 */
typedef struct {
  const void* A;       /* fp16 [M, K] activations */
  const void* packed;  /* packed weights (w4a8_pack_weights) for N x K */
  int64_t M, N, K;
  int8_t* A8;          /* int8 [M, K] codes (written) */
  void* sA;            /* fp16 [M] scales (written) */
  int32_t* rowsum;     /* int32 [M] code sums (written) */
  void* Y;             /* fp16 [M, N] output */
} w4a8_chain_link_t;

#define W4A8_CHAIN_MAX_LINKS 16
#define W4A8_CHAIN_MAX_M 32

/* Workspace bytes of w4a8_chain for these links on the current device (0 if
 * the links are invalid). */
W4A8_API size_t w4a8_chain_workspace_bytes(const w4a8_chain_link_t* links, int32_t n_links);

W4A8_API w4a8_status_t w4a8_chain(const w4a8_chain_link_t* links, int32_t n_links, void* workspace,
                                  size_t workspace_bytes, w4a8_stream_t stream);

/*
 * W4A4: 4-bit weights against 4-bit activations, the W4A4KV4 models of
 * "PrefixQuant: Static Quantization Beats Dynamic through Prefixed Outliers
 * in LLMs" (Key Findings), which quantizes activations per tensor with a
 * static scale once the outlier tokens are prefixed. The pages give no code
 * range or storage for the 4-bit activations; this library uses the 8-bit
 * scheme with the symmetric 4-bit range:
 *   A4[m,k] = clamp(rint(A[m,k] / float(s)), -7, 7)   (IEEE fp32 divide, ties to even)
 * stored two codes per byte: byte j of token m holds code 2j in bits 0-3 and
 * code 2j+1 in bits 4-7 (4-bit two's complement), i.e. A4 is uint8 [M, K/2].
 * The GEMM computes exactly what w4a8_gemm computes on those codes:
 *   Y[m,n] = fp16_rn(float(sum_k A4[m,k] * W8[n,k]) * (float(sA[m]) * float(s1[n])))
 * (the tensor cores have no 4-bit integer mode: the kernel expands each
 * activation tile to int8 in shared memory).
 */

/*
 * Per-token dynamic 4-bit activations: sA[m] = fp16_rn(amax_m / 7) (IEEE
 * fp32 divide), s = sA[m] above; sA == 0 gives zero codes.
 * A: fp16 [M, K]. A4: uint8 [M, K/2] (16-byte aligned). sA: fp16 [M] (2-byte
 * aligned). rowsum: int32 [M] (4-byte aligned) or NULL, sum_k A4[m,k].
 * Limits: K % 8 == 0, 0 < K <= 65536, M >= 0 (M == 0 is a no-op).
 */
W4A8_API w4a8_status_t w4a4_quantize_act(const void* A, int64_t M, int64_t K, uint8_t* A4, void* sA,
                                         int32_t* rowsum, w4a8_stream_t stream);

/*
 * Per-tensor static 4-bit activations (PrefixQuant's scheme): one fp16 scale
 * s (device pointer, read on the device) for the whole tensor; sA[m] = s so
 * that the GEMM's per-token epilogue applies it. Other arguments and limits
 * as for w4a4_quantize_act.
 */
W4A8_API w4a8_status_t w4a4_quantize_act_static(const void* A, int64_t M, int64_t K, const void* s, uint8_t* A4,
                                                void* sA, int32_t* rowsum, w4a8_stream_t stream);

/*
 * W4A4 GEMM: A4 uint8 [M, K/2] from w4a4_quantize_act(_static) (16-byte
 * aligned), rowsum its code sums (required, as for w4a8_gemm). Other
 * arguments, the workspace and the limits as for w4a8_gemm.
 */
W4A8_API w4a8_status_t w4a4_gemm(const uint8_t* A4, const void* sA, const int32_t* rowsum, const void* packed,
                                 int64_t M, int64_t N, int64_t K, void* Y, void* workspace, size_t workspace_bytes,
                                 w4a8_stream_t stream);

/*
 * Workspace for w4a4_gemm / w4a4_gemm_ex: w4a8_gemm_workspace_bytes(M, N, K)
 * rounded up to a multiple of 256, plus M * K. Its first
 * w4a8_gemm_workspace_bytes(M, N, K) bytes follow the rules of the w4a8
 * workspace (zero-filled once by the caller, left zero-filled by every call);
 * each call expands the packed activation codes once (one small extra
 * kernel) into the workspace's LAST M * K bytes (from a 256-byte boundary),
 * which need no particular contents, instead of inside the GEMM once per
 * output tile. A workspace of the returned size serves every M' <= M,
 * N' <= N, K' <= K. With a workspace too small for that scratch the GEMM
 * expands the codes itself in shared memory (same results, slower).
 */
W4A8_API size_t w4a4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* w4a4_gemm with the output choice and overrides of w4a8_gemm_ex. */
W4A8_API w4a8_status_t w4a4_gemm_ex(const uint8_t* A4, const void* sA, const int32_t* rowsum, const void* packed,
                                    int64_t M, int64_t N, int64_t K, void* Y, int32_t* acc, void* workspace,
                                    size_t workspace_bytes, const w4a8_gemm_opts_t* opts, w4a8_stream_t stream);

/*
 * Lookup-table weight-only GEMM (the LUT-quantized GEMM of "Fast Matrix
 * Multiplications for Lookup Table-Quantized LLMs", FLUTE, abstract): every
 * weight is a 4-bit index q into a 16-entry fp16 table T (NormalFloat-style
 * tables, for instance), with one fp16 scale s per output channel and group
 * of 128 inputs; the activations stay fp16. The pages fix no arithmetic;
 * this library computes
 *   W[n,k] = fp16_rn(float(T[q[n,k]]) * float(s[n, k/128]))   (exact product, one rounding)
 *   Y[m,n] = fp16_rn(sum_k A[m,k] * W[n,k])
 * with the products exact and the sum accumulated in fp32 in an unspecified
 * order (so within K * 2^-23 * sum_k |A W| of the exact sum).
 *
 * Packed blob, little-endian: header (64 bytes: u32 magic "W4LT", u32 version
 * 1, i64 N, i64 K, i32 group, u32 tile bytes 8448, u64 byte offset of the
 * table, zeros); (N/128) x (K/128) tiles of 8448 bytes, tile (nt, kt) at
 * 64 + (nt * K/128 + kt) * 8448: 8192 index bytes, byte j of row r's 64 bytes
 * holding the indices of in-tile k = 2j (bits 0-3) and k = 2j+1 (bits 4-7),
 * the row's 16-byte vector c at (c * 128 + r) * 16; then the 128 fp16 row
 * scales of group kt (row r at 8192 + 2r); after the tiles the 16 fp16 table
 * entries, zero padded to 64 bytes.
 */

/* Size in bytes of the lookup-table blob for an N x K weight (0 if unsupported). */
W4A8_API size_t w4lut_packed_bytes(int64_t N, int64_t K, int32_t group);

/*
 * Packs q (uint8 [N, K], one index 0..15 per byte, 16-byte aligned), s (fp16
 * [N, K/128], 2-byte aligned) and table (16 fp16 values, 2-byte aligned) into
 * the blob above. An index above 15 is reported as W4A8_DEVERR_PACK_RANGE in
 * the device error word (only its low 4 bits are packed). Limits: group == 128, N % 128 == 0, K % 128 == 0,
 * 0 < K <= 65536; packed_bytes >= w4lut_packed_bytes(N, K, group).
 */
W4A8_API w4a8_status_t w4lut_pack_weights(const uint8_t* q, const void* s, const void* table, int64_t N, int64_t K,
                                          int32_t group, void* packed, size_t packed_bytes, w4a8_stream_t stream);

/*
 * Y fp16 [M, N] = the lookup-table GEMM of A (fp16 [M, K], 16-byte aligned)
 * with the blob. workspace: as for w4a8_gemm, sized by
 * w4a8_gemm_workspace_bytes(M, N, K) (its partial sums hold fp32 here).
 * Limits as for w4a8_gemm.
 */
W4A8_API w4a8_status_t w4lut_gemm(const void* A, const void* packed, int64_t M, int64_t N, int64_t K, void* Y,
                                  void* workspace, size_t workspace_bytes, w4a8_stream_t stream);

/*
 * w4lut_gemm with overrides (block_m 0, 16 or 32 only): exactly one of Y and
 * acc (fp32 [M, N], the sums before the rounding to fp16) must be non-NULL.
 */
W4A8_API w4a8_status_t w4lut_gemm_ex(const void* A, const void* packed, int64_t M, int64_t N, int64_t K, void* Y,
                                     float* acc, void* workspace, size_t workspace_bytes,
                                     const w4a8_gemm_opts_t* opts, w4a8_stream_t stream);

/*
 * 3-bit lookup-table weights ("Fast Matrix Multiplications for Lookup
 * Table-Quantized LLMs", abstract: bit widths that do not divide a byte):
 * the same GEMM with an 8-entry fp16 table and indices 0..7. Blob,
 * little-endian: header as above with magic "W3LT" and tile bytes 6400;
 * (N/128) x (K/128) tiles of 6400 bytes, tile (nt, kt) at 64 + (nt * K/128 +
 * kt) * 6400: per row three 16-byte bit planes, plane c (bit c of the row's
 * 128 indices; bit kk of the plane = bit kk % 8 of byte kk / 8 is bit c of
 * the index at in-tile k = kk) at (c * 128 + r) * 16; then the 128 fp16 row
 * scales (row r at 6144 + 2r); after the tiles the 8 fp16 table entries,
 * zero padded to 64 bytes. Entry points as for the 4-bit table (q holds one
 * index 0..7 per byte; table holds 8 fp16 values). An index above 7 is
 * reported as W4A8_DEVERR_PACK_RANGE in the device error word (only its low
 * 3 bits are packed, which selects a different table entry).
 */
W4A8_API size_t w4lut3_packed_bytes(int64_t N, int64_t K, int32_t group);
W4A8_API w4a8_status_t w4lut3_pack_weights(const uint8_t* q, const void* s, const void* table, int64_t N, int64_t K,
                                           int32_t group, void* packed, size_t packed_bytes, w4a8_stream_t stream);
W4A8_API w4a8_status_t w4lut3_gemm(const void* A, const void* packed, int64_t M, int64_t N, int64_t K, void* Y,
                                   void* workspace, size_t workspace_bytes, w4a8_stream_t stream);
W4A8_API w4a8_status_t w4lut3_gemm_ex(const void* A, const void* packed, int64_t M, int64_t N, int64_t K, void* Y,
                                      float* acc, void* workspace, size_t workspace_bytes,
                                      const w4a8_gemm_opts_t* opts, w4a8_stream_t stream);

/*
 * 4-bit KV cache and decode attention over it (the KV4 of W4A8KV4,
 * "QServe/QoQ" abstract on the lmdeploy issue "[Feature] Support W4A8KV4
 * Quantization(QServe/QoQ)", Motivation: 4-bit KV cache, memory-bound fused
 * attention; "PrefixQuant ...", Key Findings: W4A4KV4). The pages fix no
 * format or arithmetic; this library's:
 *
 * Cached vector (one token of one kv head, D = 128 values): on the range
 * widened to include zero, lo = min(min x, 0), hi = max(max x, 0),
 *   s = fp16_rn((hi - lo) / 15),  z = clamp(rint(-lo / s), 0, 15),
 *   code = clamp(rint(x / s) + z, 0, 15)
 * (fp32, IEEE divides, ties to even; s == 0 gives z = 0 and zero codes);
 * dequantized value (code - z) * s. Stored as 64 code bytes (element 2i in
 * bits 0-3 of byte i, 2i+1 in bits 4-7) and one 32-bit parameter word: fp16 s
 * in bits 0-15, fp16 z in bits 16-31. A static per-tensor scheme is the same
 * format with one (s, z) for every vector.
 *
 * Cache layout: codes uint8 [B, Hkv, Lmax, 64], parameter words uint32
 * [B, Hkv, Lmax]; sequence b holds its tokens at positions 0 .. L_b - 1.
 *
 * Decode attention, one query token per sequence: query head h reads kv head
 * h / (Hq / Hkv);
 *   s_j = scale * (s_j^K * sum_d q[d] (code^K_jd - z^K_j)),  j < L_b
 *   Y[b, h] = fp16_rn(sum_j softmax(s)_j (code^V_j - z^V_j) s^V_j)
 * in fp32 (so within the fp32 evaluation bound of the exact result plus half
 * an fp16 ulp); L_b == 0 gives Y = 0.
 */

/* Quantizes n contiguous fp16 vectors X [n, 128] (16-byte aligned) into codes
 * [n, 64] (16-byte aligned) and parameter words [n] (4-byte aligned). D must
 * be 128. */
W4A8_API w4a8_status_t w4kv_quantize(const void* X, int64_t n, int32_t D, uint8_t* codes, uint32_t* params,
                                     w4a8_stream_t stream);

/* Appends one token per (sequence, kv head): K_new and V_new fp16 [B, Hkv,
 * 128] are quantized into the caches at position positions[b] (int32 [B],
 * device memory). A position outside [0, Lmax) is skipped and recorded as
 * W4A8_DEVERR_KV_RANGE in the device error word. */
W4A8_API w4a8_status_t w4kv_append(const void* K_new, const void* V_new, const int32_t* positions, int64_t B,
                                   int64_t Hkv, int64_t Lmax, int32_t D, uint8_t* k_codes, uint32_t* k_params,
                                   uint8_t* v_codes, uint32_t* v_params, w4a8_stream_t stream);

/* Workspace bytes of w4kv_attention_decode (0 if the shape is unsupported):
 * one partial result (2 + 128 floats) per (sequence, query head, chunk of 128
 * cache positions). */
W4A8_API size_t w4kv_attention_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Lmax, int32_t D);

/*
 * Y fp16 [B, Hq, 128] (16-byte aligned) = decode attention of q fp16 [B, Hq,
 * 128] (16-byte aligned) over the caches (codes 16-byte, parameter words
 * 4-byte aligned) with lengths seq_lens (int32 [B], device memory; a length
 * outside [0, Lmax] is clamped and recorded as W4A8_DEVERR_KV_RANGE).
 * Limits: D == 128, Hkv >= 1, Hq % Hkv == 0, Hq <= 65536, 1 <= Lmax <= 2^24,
 * B <= 65535. workspace: 256-byte aligned, at least
 * w4kv_attention_workspace_bytes(...) bytes, any contents (it holds the
 * chunks' partial results between the call's two kernels). Calls that share a
 * workspace must not overlap on the GPU. Both contractions run on tensor
 * cores with fp32 accumulation: the scores from fp16 q and the exact small
 * integers code - z, the weighted values from the same integers (bf16) and
 * the softmax weights split into three bf16 terms (relative error below
 * 2^-24), within the fp32 evaluation bound above.
 */
W4A8_API w4a8_status_t w4kv_attention_decode(const void* q, const uint8_t* k_codes, const uint32_t* k_params,
                                             const uint8_t* v_codes, const uint32_t* v_params,
                                             const int32_t* seq_lens, int64_t B, int64_t Hq, int64_t Hkv,
                                             int64_t Lmax, int32_t D, float scale, void* out, void* workspace,
                                             size_t workspace_bytes, w4a8_stream_t stream);

/*
 * Allocation-free GEMM: the same computation and results as w4a8_gemm, for
 * callers that cannot hand the library a workspace. This entry point has no
 * counterpart in the papers; it exists for deployment. Typical callers: a
 * plugin or custom operator inside a host engine that plans all device
 * memory itself and gives the operator no scratch buffer, or a serving loop
 * that must not touch the device allocator once it has started.
 *
 * Instead of a caller-provided workspace it uses one scratch array compiled
 * into the library (a file-scope __device__ array of
 * W4A8_NOALLOC_SCRATCH_BYTES = 8 MiB, 256-byte aligned). Every GPU that
 * loads the library holds that array until the process exits.
 *  - Set-up: the first call on a device (with that device current) looks up
 *    the array's device address with cudaGetSymbolAddress and caches it.
 *    Make that first call before any stream capture on the device.
 *  - Each call clears the part of the array it needs (cudaMemsetAsync on
 *    `stream`) and then launches the GEMM; it calls no cudaMalloc, cudaFree
 *    or other allocating routine.
 *  - The array is shared by every call on a device and keeps the last call's
 *    contents: calls whose GPU work overlaps in time (different streams
 *    without ordering between them) race on it and give wrong results.
 *  - Shapes whose scratch need, w4a8_gemm_workspace_bytes(M, N, K), exceeds
 *    W4A8_NOALLOC_SCRATCH_BYTES are rejected with W4A8_ERR_WORKSPACE and
 *    nothing is launched (every M <= 32 fits for N <= 49152; M = 64 fits for
 *    N <= 32640; larger M or N may not).
 * Arguments, layouts and the other limits are those of w4a8_gemm.
 */
#define W4A8_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
W4A8_API w4a8_status_t w4a8_gemm_noalloc(const int8_t* A8, const void* sA, const int32_t* rowsum, const void* packed,
                                         int64_t M, int64_t N, int64_t K, void* Y, w4a8_stream_t stream);

/*
 * Synchronizes `stream`, then stores the current device's error word in
 * *code (W4A8_DEVERR_*; 0 = no kernel gave up a wait). Returns W4A8_ERR_CUDA
 * if the synchronization itself fails. The word stays set until cleared.
 */
W4A8_API w4a8_status_t w4a8_get_device_error(w4a8_stream_t stream, int32_t* code);

/* Resets the current device's error word to 0 (stream-ordered). */
W4A8_API w4a8_status_t w4a8_clear_device_error(w4a8_stream_t stream);

/*
 * Failure-path self-test (no counterpart in the papers; it exercises the
 * library's own failure detection). Launches one warp that waits on an
 * mbarrier nothing ever completes, with the same bounded wait every kernel of
 * the library uses but a limit of `limit_ns` (clamped to [1 us, 2 s]). The
 * wait gives up, records W4A8_DEVERR_SELFTEST_WAIT in the device error word
 * (unless it already holds a code) and the kernel returns: no fault, no hang,
 * and the context stays usable. Read the result with w4a8_get_device_error
 * and reset it with w4a8_clear_device_error.
 */
W4A8_API w4a8_status_t w4a8_selftest_bounded_wait(int64_t limit_ns, w4a8_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A8_H_ */

// prefill_tc.cu -- causal chunked-prefill attention over the paged KV cache (rotated INT4 or
// NVFP4) on the 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory),
// sm_100a.
//
// Method: "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化"
// (youngju.dev): section "KVキャッシュこそが本当のボトルネックである理由" (attention runs
// over the paged cache in serving engines) and "回転のトリック — ブロック対角アダマール"
// (the orthonormal rotation keeps q.k, so attention runs in the rotated domain and the output
// is rotated back).  A chunk of C prompt tokens of a sequence, already appended, attends the
// cache causally: query i of the chunk (position L - C + i) sees positions 0..L - C + i.
//
// Work decomposition.  A CTA takes 128 query rows of one (sequence, KV head): 128 / G
// consecutive chunk tokens times the G query heads of the KV head.  Row r is lane r of tensor
// memory.  The CTA's 22 warps specialise and hand work to one another through mbarriers, so
// the softmax, the code expansion and the tensor cores overlap instead of taking turns:
//   warps 0-15   softmax: warps q, q + 4, q + 8, q + 12 all read the lanes of rows 32q..,
//                warp q + 4j the j-th 32 columns of each tile and of O (four threads per
//                row: the special-function unit's exponentials and the other phases of
//                the warps sharing an SMSP overlap better than with two);
//   warps 16-19  expansion: the K and V codes of a tile into the MMA operand tiles, plus
//                their scales;
//   warp 20      one lane issues the MMAs: QK^T of tile t, then PV of tile t - 1;
//   warp 21      reads the page table and issues the bulk copies of the raw page data.
// Tensor-core time per instruction hardly depends on N up to 128 here, so the tiles are as
// wide as the accumulators allow (S of two tiles, O and q~ fill the 512 TMEM columns).
// S (tensor memory), the K and V operand tiles and the scales are double-buffered by tile
// parity; the raw page data streams through four slots (three on NVFP4).  The causal KV
// range is cut into tiles of 128 tokens, whose pages are bulk-copied (cp.async.bulk, 1-D,
// no multicast).
//   QK^T  tcgen05.mma kind::f16, M = 128 rows, N = 128 tokens, K = 128 channels: A = q' cut
//         into fp16 hi + lo parts (q' * 2^14 / M_r, M_r the power of two >= max |q'_r|), held
//         in tensor memory for the whole CTA; B = the K codes as exact fp16 integers in shared
//         memory; both parts accumulate into one fp32 tile S in tensor memory.  The K scale
//         and the row's M_r / 2^14 multiply the scores.
//   softmax  each thread loads its quarter row of S (tcgen05.ld), applies the causal mask;
//         the four quarters' maxima meet in shared memory; the row keeps an online maximum m
//         and sum l in the log2 domain.  The frame m moves only when a score exceeds it by
//         more than 8 (then the row of O is rescaled in tensor memory), so
//         p = 2^(score - m) <= 256 and the rescale is rare.
//   PV    tcgen05.mma kind::f16 in bf16, M = 128 rows, N = 128 channels, K = 128 tokens: A =
//         P' = p * s_v (the V scale folded into the probabilities) as bf16 hi + lo parts (bf16
//         keeps fp32's range, so P' <= 256 * s_v cannot overflow), written by each softmax
//         thread over the S columns it has just read; B = the V codes as exact bf16 integers,
//         read channel-major from shared memory; the accumulator O stays in tensor memory.
// With both A operands in tensor memory the tensor cores read only K and V from shared
// memory, whose bandwidth the MMAs would otherwise share with the expansion.
// The end: each thread loads its quarter row of O, divides by l, applies the inverse block
// Hadamard (stages inside a quarter in registers, the two stages across quarters through
// shared memory), times c_b, stores fp16.  On the NVFP4 cache the expansion dequantises K
// and V exactly to fp16 (block scales folded in), and PV runs in fp16 with P' = p.
//
// Shared-memory operands use the 128-byte swizzle of the tensor core's canonical layouts: 8
// rows of 128 bytes per 1024-byte atom, the 16-byte chunk index XOR the row within the atom.
// Every wait is bounded (2 s); a wait that gives up flags KVQ_DEV_TIMEOUT, and the CTA
// still waits (bounded) for its copies and MMAs before releasing tensor memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>
#include <stdint.h>

#include "../../include/kvq.h"
#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kD = 128;
constexpr int kRowsT = 128;     // query rows per CTA (tensor-memory lanes)
constexpr int kTokT = 128;      // KV tokens per tile
constexpr int kSoftWarps = 16;  // warps q, q + 4, q + 8, q + 12 share the rows of TMEM lanes 32q..
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kExpWarp0 = 16;   // warps 16-19 expand K and V codes
constexpr int kExpWarps = 4;
constexpr int kExpThreads = 32 * kExpWarps;
constexpr int kMmaWarp = 20;    // issues the tcgen05 MMAs
constexpr int kProdWarp = 21;   // reads the page table and issues the bulk copies
constexpr int kThreadsT = 704;
constexpr uint64_t kWaitT = 2000000000ull;
constexpr float kLazyT = 8.0f;  // frame slack in log2 units: p <= 2^8 between rescales
constexpr unsigned kFullT = 0xffffffffu;
// Tensor-memory columns: S of tiles t even / odd [0, 128) / [128, 256), where P' of the tile
// replaces S once read; O [256, 384); q~ hi [384, 448) and lo [448, 512) (fp16 pairs).
constexpr int kTmemCols = 512;
constexpr int kColO = 256;
constexpr int kColQh = 384;
constexpr int kColQl = 448;

// Shared-memory map (bytes from a 1024-byte aligned base).
constexpr int kKs = 0;                          // [2 buffers][2 kb][128 tokens][128 B] fp16 K codes
constexpr int kKsBuf = 2 * kTokT * 128;
// q~ passes through the K buffers on its way to tensor memory (before any K is expanded),
// and the end exchanges the four parts of O there (after the last QK^T).
constexpr int kQh = kKs;                        // [2 kb][128 rows][128 B] fp16 q~ hi
constexpr int kQl = kQh + 2 * kRowsT * 128;     // same, lo
constexpr int kVs = kKs + 2 * kKsBuf;           // [2 buffers][2 nb][128 tokens][128 B] bf16 V codes
constexpr int kVsBuf = 2 * kTokT * 128;
constexpr int kRing = kVs + 2 * kVsBuf;         // raw page-data slots, see TcFmt
constexpr int kBarFull = 0, kBarEmpty = 4, kBarKReady = 8, kBarVReady = 10, kBarSFull = 12,
              kBarSFree = 14, kBarPReady = 16, kBarPVDone = 17, kNumBars = 19;
static_assert(kQl + 2 * kRowsT * 128 <= kVs, "q~ staging fits the K buffers");

// What depends on the cache format: a (token, KV head) row is 132 B in INT4 ([64 B K codes]
// [64 B V codes] and one fp16 scale each) and 144 B in NVFP4 (the same codes, then 8 E4M3
// block scales each); the raw slots (4 INT4, 3 NVFP4) and the rest of the map follow.
template <bool FP4>
struct TcFmt {
  static constexpr int kRowB = FP4 ? 144 : 132;
  static constexpr int kScB = FP4 ? 8 : 2;        // scale bytes per token, K or V
  static constexpr int kStages = FP4 ? 3 : 4;
  static constexpr int kSlot = kTokT * kRowB;     // [128 token rows] in page-block layout
  static constexpr int kScl = kRing + kStages * kSlot;  // K [2][128], V [2][128] fp32 multipliers
  static constexpr int kSfr = kScl + 4 * kTokT * 4;     // row scales [128] fp32
  static constexpr int kRed = kSfr + kRowsT * 4;        // maxima [2][4][128], sums [4][128]
  static constexpr int kBar = kRed + 12 * kRowsT * 4;   // mbarriers, see kBar* above
  static constexpr int kTmemSlot = kBar + kNumBars * 8; // tensor-memory base address
  static constexpr int kPreq = kTmemSlot + 16;          // query-block prefix [batch + 1]
  static_assert(kStages <= 4, "four full / empty barriers");
  static_assert(kPreq + 4097 * 4 + 1024 + 1024 <= 232448, "shared memory of the largest batch");
};

// Instruction descriptors (kind::f16): fp32 accumulator, M = 128.
//   QK^T: A, B fp16, both K-major, N = 128.  PV: A, B bf16 (INT4) or fp16 (NVFP4), A K-major,
//   B MN-major, N = 128.
constexpr uint32_t kIdescQK = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((128u >> 3) << 17) |
                              ((128u >> 4) << 24);
constexpr uint32_t kIdescPVh = (1u << 4) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// Byte offset of the 16-byte chunk `chunk` of row `row` in a 128-byte swizzled operand.
__device__ __forceinline__ uint32_t sw_off(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// The raw slot holds virtual pages of SEFF = min(S, 128) token rows in the pool's block layout
// [K codes][V codes][K scales][V scales].  Copying a tile takes two steps so that the page-
// table read can be issued well before the copies: tile_page reads this lane's page id of
// tile t of sequence b (lane i the tile's i-th page when pages are shorter than a tile, else
// every lane the one page); issue_tile_pages checks it (an id out of range flags
// KVQ_DEV_BAD_PAGE and reads page 0) and starts the copies into a slot with completion on its
// barrier.
template <int SEFF, bool FP4>
__device__ __forceinline__ int tile_page(int t, int b, int L, int lane, const PrefillParams& p) {
  const int sh = p.page_shift;
  const int t0 = t * kTokT;
  const int t1 = min(t0 + kTokT, L);  // > t0
  const int npg = (SEFF < kTokT || p.page_size == kTokT) ? ((t1 - 1) >> sh) - (t0 >> sh) + 1 : 1;
  if (npg > 1 && lane >= npg) return 0;
  return __ldg(p.page_table + static_cast<size_t>(b) * p.max_pages_per_seq + (t0 >> sh) + (npg > 1 ? lane : 0));
}

template <int SEFF, bool FP4>
__device__ __forceinline__ void issue_tile_pages(int t, int h, int L, int pid, uint32_t slot, uint32_t bar,
                                                 int lane, uint64_t pol, const PrefillParams& p) {
  const int S = p.page_size, sh = p.page_shift;
  const int t0 = t * kTokT;
  const int t1 = min(t0 + kTokT, L);  // > t0
  if (pid < 0 || pid >= p.num_pages) {
    if (lane == 0 || SEFF < kTokT || S == kTokT) atomicOr(p.status, KVQ_DEV_BAD_PAGE_BIT);
    pid = 0;
  }
  if (SEFF < kTokT || S == kTokT) {
    const uint32_t blk_bytes = static_cast<uint32_t>(S) * TcFmt<FP4>::kRowB;
    const int npg = ((t1 - 1) >> sh) - (t0 >> sh) + 1;
    if (lane == 0) mbar_arrive_expect_tx(bar, npg * blk_bytes);
    __syncwarp();
    if (lane < npg)
      bulk_copy_g2s(slot + lane * blk_bytes,
                    p.pool_layer + (static_cast<size_t>(pid) * p.num_kv_heads + h) * blk_bytes,
                    blk_bytes, bar, pol);
  } else {
    // Pages of 128+ tokens: the tile is part of one page; lanes 0-3 copy its K codes, V
    // codes, K scales and V scales.
    constexpr int sb = TcFmt<FP4>::kScB;
    const size_t blk_bytes = static_cast<size_t>(S) * TcFmt<FP4>::kRowB;
    const size_t o = static_cast<size_t>(t0 & (S - 1));
    const uint8_t* blk = p.pool_layer + (static_cast<size_t>(pid) * p.num_kv_heads + h) * blk_bytes;
    const uint8_t* src = blk + o * 64;
    uint32_t dst = slot, bytes = kTokT * 64;
    if (lane == 1) { src = blk + static_cast<size_t>(S) * 64 + o * 64; dst = slot + kTokT * 64; }
    if (lane == 2) { src = blk + static_cast<size_t>(S) * 128 + o * sb; dst = slot + kTokT * 128; bytes = kTokT * sb; }
    if (lane == 3) {
      src = blk + static_cast<size_t>(S) * (128 + sb) + o * sb;
      dst = slot + kTokT * (128 + sb);
      bytes = kTokT * sb;
    }
    if (lane == 0) mbar_arrive_expect_tx(bar, TcFmt<FP4>::kSlot);
    __syncwarp();
    if (lane < 4) bulk_copy_g2s(dst, src, bytes, bar, pol);
  }
}

// Byte k of w: its two signed 4-bit codes (low nibble = even channel) as exact fp16 (lo
// half = even channel).  (w & 0x000F) ^ 0x6408 is fp16 1024 + (n ^ 8) = 1032 + n; the high
// nibble lands as 1024 + 16 (n + 8); one fma per half takes both to n.
__device__ __forceinline__ uint32_t codes_f16x2(uint32_t w, int k) {
  uint32_t x = prmt(w, 0u, static_cast<uint32_t>(k) | (static_cast<uint32_t>(k) << 8) | 0x4040u);
  x = lop3_and_xor(x, 0x00F0000Fu, 0x64806408u);
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(x) : "r"(x), "r"(0x2C003C00u), "r"(0xD480E408u));
  return x;
}

// The same as bf16: lo = word w (low nibbles), hi = w >> 4 (high nibbles at the bottom of
// each byte); (x & 0x000F000F) ^ 0x43084308 is bf16 128 + (n ^ 8) = 136 + n per half.
__device__ __forceinline__ uint32_t codes_bf16x2(uint32_t lo, uint32_t hi, int k) {
  uint32_t x = prmt(lo, hi, static_cast<uint32_t>(k) | ((4u + static_cast<uint32_t>(k)) << 8));
  x = lop3_and_xor(x, 0x000F000Fu, 0x43084308u);
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(x) : "r"(x), "r"(0x3F803F80u), "r"(0xC308C308u));
  return x;
}

// NVFP4: one byte of two E2M1 codes (low nibble first) -> fp16x2; two E4M3 bytes -> fp16x2.
// Both exact (the formats' values are fp16 values).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2_t(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
      : "=r"(r)
      : "r"(byte));
  return r;
}
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_t(uint32_t b) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(b)));
  return h;
}
__device__ __forceinline__ uint32_t hmul2_t(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// NVFP4 row half: channels 64 hf..64 hf + 63 of K (kv 0) or V (kv 1) of token row jr of a
// virtual page, dequantised to fp16 (E2M1 value x E4M3 block scale has at most 6 significant
// bits and lies in [2^-10, 2688]: exact) into row ej of a 128-byte swizzled operand tile.
// A token past the sequence's end takes scale 0, so its (arbitrary) bytes become zeros.
template <int SEFF>
__device__ __forceinline__ void expand_fp4_half(const uint8_t* pg, int jr, int kv, int hf, bool live,
                                                uint8_t* dst, int ej) {
  const uint4* src = reinterpret_cast<const uint4*>(pg + kv * SEFF * 64 + jr * 64 + 32 * hf);
  const uint4 c0 = src[0], c1 = src[1];
  const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const uint32_t sc = live ? *reinterpret_cast<const uint32_t*>(pg + SEFF * 128 + kv * SEFF * 8 + jr * 8 + 4 * hf)
                           : 0u;
  const uint32_t s01 = e4m3x2_to_f16x2_t(sc & 0xFFFFu), s23 = e4m3x2_to_f16x2_t(sc >> 16);
  const uint32_t sdup[4] = {prmt(s01, s01, 0x1010u), prmt(s01, s01, 0x3232u), prmt(s23, s23, 0x1010u),
                            prmt(s23, s23, 0x3232u)};  // blocks 4 hf .. 4 hf + 3, both halves
#pragma unroll
  for (int ch = 0; ch < 8; ch++) {  // 16-byte chunk ch = channels 64 hf + 8 ch .. + 7, block ch / 2
    uint32_t hv[4];
#pragma unroll
    for (int k = 0; k < 4; k++) hv[k] = hmul2_t(e2m1x2_to_f16x2_t(cw[ch] >> (8 * k)), sdup[ch >> 1]);
    *reinterpret_cast<uint4*>(dst + sw_off(ej, ch)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
  }
}

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

template <int G, int SEFF, bool FP4>
__global__ void __launch_bounds__(kThreadsT, 1) prefill_tc_kernel(PrefillParams p) {
  using F = TcFmt<FP4>;
  constexpr int QB = kRowsT / G;  // chunk tokens per CTA
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  float* s_kb = reinterpret_cast<float*>(smem + F::kScl);  // [2][128] K multipliers, tiles t even / odd
  float* s_vb = s_kb + 2 * kTokT;                          // [2][128] V multipliers
  float* sfr = reinterpret_cast<float*>(smem + F::kSfr);
  float* red = reinterpret_cast<float*>(smem + F::kRed);  // [tile parity][part][row] maxima
  float* lsum = red + 8 * kRowsT;                         // [part][row] final sums
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + F::kTmemSlot);
  int32_t* preq = reinterpret_cast<int32_t*>(smem + F::kPreq);
  const uint32_t bar0 = sbase + F::kBar;
  const uint32_t full_s = bar0 + 8 * kBarFull, empty_s = bar0 + 8 * kBarEmpty, kready = bar0 + 8 * kBarKReady,
                 vready = bar0 + 8 * kBarVReady, sfull = bar0 + 8 * kBarSFull,
                 sfree = bar0 + 8 * kBarSFree, pready = bar0 + 8 * kBarPReady,
                 pvdone = bar0 + 8 * kBarPVDone;
  __shared__ int warp_sum[kThreadsT / 32];
  __shared__ int running;

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  // Before griddep_wait only cu_q, seq_lens and the page table are read (inputs of this
  // call); q, the pool and out are touched after it.
  griddep_launch_dependents();
  if (tid == 0) {
    for (int k = 0; k < F::kStages; k++) {
      mbar_init(full_s + 8 * k, 1);
      mbar_init(empty_s + 8 * k, kExpThreads);
    }
    for (int k = 0; k < 2; k++) {
      mbar_init(kready + 8 * k, kExpThreads);
      mbar_init(vready + 8 * k, kExpThreads);
      mbar_init(sfull + 8 * k, 1);
      mbar_init(sfree + 8 * k, kSoftThreads);
      mbar_init(pvdone + 8 * k, 1);
    }
    mbar_init(pready, kSoftThreads);
    fence_mbar_init();
    running = 0;
  }
  __syncthreads();

  // Query blocks per sequence -> exclusive prefix preq[0..batch].
  for (int base = 0; base < p.batch; base += kThreadsT) {
    const int i = base + tid;
    int n = 0;
    if (i < p.batch) {
      const int C = __ldg(p.cu_q + i + 1) - __ldg(p.cu_q + i);
      n = C > 0 ? (C + QB - 1) / QB : 0;
    }
    int incl = n;
#pragma unroll
    for (int d = 1; d < 32; d *= 2) {
      const int y = __shfl_up_sync(kFullT, incl, d);
      if (lane >= d) incl += y;
    }
    if (lane == 31) warp_sum[w] = incl;
    __syncthreads();
    int before = running;
    for (int w2 = 0; w2 < w; w2++) before += warp_sum[w2];
    if (i < p.batch) preq[i] = before + incl - n;
    __syncthreads();
    if (tid == kThreadsT - 1) running = before + incl;
    __syncthreads();
  }
  if (tid == 0) preq[p.batch] = running;
  __syncthreads();

  const int nblk = preq[p.batch];
  const int qbg = blockIdx.x / p.num_kv_heads, h = blockIdx.x - qbg * p.num_kv_heads;
  if (qbg >= nblk) return;  // the whole CTA
  int lo = 0, hi = p.batch;  // preq[lo] <= qbg < preq[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (preq[mid] <= qbg) lo = mid; else hi = mid;
  }
  const int b = lo, qb = qbg - preq[b];
  const int cq0 = __ldg(p.cu_q + b);
  const int C = __ldg(p.cu_q + b + 1) - cq0;
  const int cap = p.max_pages_per_seq * p.page_size;
  const int L = __ldg(p.seq_lens + b);
  if (L > cap || C > L || cq0 < 0 || cq0 + C > p.total_q) {
    if (tid == 0) atomicOr(p.status, KVQ_DEV_BAD_POS_BIT);
    return;
  }
  const int tok_first = qb * QB;                      // first chunk token of the CTA
  const int tok_last = min(C, tok_first + QB) - 1;    // last valid one
  const int ntile = (L - C + tok_last) / kTokT + 1;   // >= 1
  const uint64_t pol = l2_policy_evict_first();

  // Tensor memory for S and O (one warp allocates; the address goes through shared memory).
  if (w == 0) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  griddep_wait();
  // The producer warp starts the copies of the first tiles, one per raw slot.
  if (w == kProdWarp) {
    for (int t = 0; t < F::kStages && t < ntile; t++)
      issue_tile_pages<SEFF, FP4>(t, h, L, tile_page<SEFF, FP4>(t, b, L, lane, p), sbase + kRing + t * F::kSlot,
                             full_s + 8 * t, lane, pol, p);
  }

  // q rows: softmax warp w rotates and scales rows 8w..8w+7 (lane: channels 4 lane..
  // 4 lane + 3) and stores q~ = q' * 2^14 / M as fp16 hi + lo parts into swizzled staging
  // tiles, from which each softmax thread moves its part of its row into tensor memory.
  if (w < kSoftWarps) {
    for (int rr = 0; rr < kRowsT / kSoftWarps; rr++) {
      const int row = (kRowsT / kSoftWarps) * w + rr;
      const int ti = tok_first + row / G, gq = row % G;
      float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (ti < C) {
        const __half* qrow = p.q + ((static_cast<size_t>(cq0) + ti) * p.num_kv_heads * G + h * G + gq) * kD;
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qrow) + lane);
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
        const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
        x[0] = a.x; x[1] = a.y; x[2] = c.x; x[3] = c.y;
      }
      if (p.hadamard_block > 1) {
        const float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
        x[0] = a0 + a2; x[2] = a0 - a2; x[1] = a1 + a3; x[3] = a1 - a3;
#pragma unroll
        for (int st = 0; st < 5; st++) {
          if ((4 << st) < p.hadamard_block) {
            const float sgn = ((lane >> st) & 1) ? -1.0f : 1.0f;
#pragma unroll
            for (int e = 0; e < 4; e++) x[e] = __fmaf_rn(x[e], sgn, __shfl_xor_sync(kFullT, x[e], 1 << st));
          }
        }
      }
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; e++) {
        x[e] = x[e] * p.cb * p.q_scale;
        amax = fmaxf(amax, fabsf(x[e]));
      }
#pragma unroll
      for (int d = 1; d < 32; d *= 2) amax = fmaxf(amax, __shfl_xor_sync(kFullT, amax, d));
      float M = 1.0f;
      if (amax > 1e-30f) {
        const uint32_t bits = __float_as_uint(amax);
        M = (bits & 0x7FFFFFu) ? __uint_as_float((bits & 0x7F800000u) + 0x00800000u) : amax;
      }
      const float inv = __fdiv_rn(16384.0f, M);  // exact: powers of two
      __half hv[4], lv[4];
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const float t = x[e] * inv;
        hv[e] = __float2half_rn(t);
        lv[e] = __float2half_rn(t - __half2float(hv[e]));
      }
      // Channels 4 lane..: K-block lane / 16, chunk (lane % 16) / 2, bytes 8 (lane % 2).
      const uint32_t off = (lane >> 4) * (kRowsT * 128) + sw_off(row, (lane & 15) >> 1) + 8 * (lane & 1);
      *reinterpret_cast<uint2*>(smem + kQh + off) = make_uint2(pack_half2(hv[0], hv[1]), pack_half2(hv[2], hv[3]));
      *reinterpret_cast<uint2*>(smem + kQl + off) = make_uint2(pack_half2(lv[0], lv[1]), pack_half2(lv[2], lv[3]));
      if (lane == 0) sfr[row] = M * (1.0f / 16384.0f);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool dead = false;
  // q~ into tensor memory, the A operand of QK^T: softmax thread (row, part) moves channels
  // 32 part..32 part + 31 of its row, hi and lo parts, as fp16 pairs (16 columns each).
  if (w < kSoftWarps) {
    const int row = 32 * (w & 3) + lane, part = w >> 2;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * (w & 3)) << 16);
#pragma unroll
    for (int hl = 0; hl < 2; hl++) {
      uint32_t r[16];
      const uint8_t* src = smem + (hl ? kQl : kQh) + (part >> 1) * (kRowsT * 128);
#pragma unroll
      for (int c = 0; c < 4; c++) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + sw_off(row, 4 * (part & 1) + c));
        r[4 * c] = v.x; r[4 * c + 1] = v.y; r[4 * c + 2] = v.z; r[4 * c + 3] = v.w;
      }
      tmem_st16(lane_addr + (hl ? kColQl : kColQh) + 16 * part, r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (w < kSoftWarps) {
    // ---------------------------------------------------------------- softmax warps --
    // This thread's row and part: tokens 32 part..32 part + 31 of every tile, channels
    // 32 part..32 part + 31 of O.  The four parts of a row are warps q, q + 4, q + 8, q + 12
    // (q = the row's TMEM lane quarter); they meet at a 128-thread named barrier.
    const int quarter = w & 3, part = w >> 2;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
    const int row = 32 * quarter + lane;
    const int ti_row = tok_first + row / G;
    const bool row_valid = ti_row < C;
    // The row's position: it sees tokens 0..rpos.  Padding rows past the chunk take the last
    // token's, so that every tile token at or beyond L is masked for them too.
    const int rpos = min(L - C + ti_row, L - 1);
    const float sf = sfr[row];
    float m = -CUDART_INF_F, l = 0.0f;
    for (int t = 0; t < ntile; t++) {
      const uint32_t par = static_cast<uint32_t>((t >> 1) & 1);
      if (!dead && !mbar_wait_bounded(sfull + 8 * (t & 1), par, kWaitT)) dead = true;
      if (!dead && !mbar_wait_bounded(kready + 8 * (t & 1), par, kWaitT)) dead = true;
      tc_fence_after();
      // u = S * s_k for this thread's 32 tokens, in pairs.  The row scale sf > 0 commutes
      // with the maximum, so the score sf * u is formed only inside the exponent.
      uint32_t raw[32];
      tmem_ld32(lane_addr + kTokT * (t & 1) + 32 * part, raw);
      tmem_wait_ld();
      uint64_t u2[16];
      const float4* s_k4 = reinterpret_cast<const float4*>(s_kb + (t & 1) * kTokT + 32 * part);
#pragma unroll
      for (int e4 = 0; e4 < 8; e4++) {
        const float4 k4 = s_k4[e4];
        u2[2 * e4] = f2_mul(f2_pack(__uint_as_float(raw[4 * e4]), __uint_as_float(raw[4 * e4 + 1])),
                            f2_pack(k4.x, k4.y));
        u2[2 * e4 + 1] = f2_mul(f2_pack(__uint_as_float(raw[4 * e4 + 2]), __uint_as_float(raw[4 * e4 + 3])),
                                f2_pack(k4.z, k4.w));
      }
      // S buffer t & 1 and the K scales of tile t are free for tile t + 2.
      tc_fence_before();
      if (!dead) mbar_arrive(sfree + 8 * (t & 1));
      // Tiles wholly before the CTA's first row need no causal mask (they hold no token at or
      // beyond L either).
      if (t * kTokT + kTokT - 1 > L - C + tok_first) {
#pragma unroll
        for (int e2 = 0; e2 < 16; e2++) {
          float2 v = f2_unpack(u2[e2]);
          const int pos = t * kTokT + 32 * part + 2 * e2;
          if (pos > rpos) v.x = -CUDART_INF_F;
          if (pos + 1 > rpos) v.y = -CUDART_INF_F;
          u2[e2] = f2_pack(v.x, v.y);
        }
      }
      float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
#pragma unroll
      for (int e2 = 0; e2 < 16; e2++) {
        const float2 v = f2_unpack(u2[e2]);
        mx0 = fmaxf(mx0, v.x);
        mx1 = fmaxf(mx1, v.y);
      }
      float mx = fmaxf(mx0, mx1) * sf;
      // The row's maximum over its four parts (the exchange slots alternate with the tile's
      // parity, so a slot is rewritten only after every part has passed the next barrier).
      red[((t & 1) * 4 + part) * kRowsT + row] = mx;
      asm volatile("bar.sync %0, 128;" ::"r"(1 + quarter) : "memory");
#pragma unroll
      for (int q2 = 1; q2 < 4; q2++) mx = fmaxf(mx, red[((t & 1) * 4 + (part ^ q2)) * kRowsT + row]);
      // Lazy frame: move m only when a score exceeds it by more than kLazyT.
      float alpha = 1.0f;
      const bool move = mx > m + kLazyT;
      if (move) {
        alpha = m == -CUDART_INF_F ? 0.0f : ex2_approx(m - mx);
        l *= alpha;
        m = mx;
      }
      // p = 2^(sf * u - m); ex2(-inf) = +0, so masked scores need no test.
      const uint64_t sf2 = f2_pack(sf, sf), nm2 = f2_pack(-m, -m);
      uint64_t ps2 = f2_pack(0.0f, 0.0f);
#pragma unroll
      for (int e2 = 0; e2 < 16; e2++) {
        const float2 a = f2_unpack(f2_fma(u2[e2], sf2, nm2));
        u2[e2] = f2_pack(ex2_approx(a.x), ex2_approx(a.y));
        ps2 = f2_add(ps2, u2[e2]);
      }
      const float2 psum = f2_unpack(ps2);
      l += psum.x + psum.y;
      // PV of tile t - 1 reads P' and accumulates O: wait for it before touching either.
      if (t > 0 && !dead &&
          !mbar_wait_bounded(pvdone + 8 * ((t - 1) & 1), static_cast<uint32_t>(((t - 1) >> 1) & 1), kWaitT))
        dead = true;
      tc_fence_after();
      // Rescale this thread's part of O when a row of the warp moved after its first tile.
      if (__any_sync(kFullT, move && alpha != 0.0f) && t > 0) {
        uint32_t o[32];
        tmem_ld32(lane_addr + kColO + 32 * part, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e++) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st32(lane_addr + kColO + 32 * part, o);
      }
      // P' = p * s_v as hi + lo pairs over this thread's own S columns (the A operand of PV):
      // columns 32 part + [0, 16) hi, + [16, 32) lo; bf16 on INT4, fp16 on NVFP4 (where V
      // carries its scales and s_v = 1).  The V scales of tile t come with vready.
      if (!dead && !mbar_wait_bounded(vready + 8 * (t & 1), par, kWaitT)) dead = true;
      {
        const float4* s_v4 = reinterpret_cast<const float4*>(s_vb + (t & 1) * kTokT + 32 * part);
        uint32_t pp[32];
#pragma unroll
        for (int c4 = 0; c4 < 8; c4++) {
          const float4 va = s_v4[c4];
          const uint64_t x2[2] = {f2_mul(u2[2 * c4], f2_pack(va.x, va.y)),
                                  f2_mul(u2[2 * c4 + 1], f2_pack(va.z, va.w))};
#pragma unroll
          for (int j = 0; j < 2; j++) {
            const float2 x = f2_unpack(x2[j]);
            if constexpr (FP4) {  // P' = p <= 256 as fp16 hi + lo
              const uint32_t hi2 = pack_f16x2(x.x, x.y);
              const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi2));
              const float2 lo = f2_unpack(f2_sub(x2[j], f2_pack(hf.x, hf.y)));
              pp[2 * c4 + j] = hi2;
              pp[16 + 2 * c4 + j] = pack_f16x2(lo.x, lo.y);
            } else {
              const uint32_t hi2 = pack_bf16x2(x.x, x.y);
              const float2 lo = f2_unpack(f2_sub(x2[j], f2_pack(bf16_lo(hi2), bf16_hi(hi2))));
              pp[2 * c4 + j] = hi2;
              pp[16 + 2 * c4 + j] = pack_bf16x2(lo.x, lo.y);
            }
          }
        }
        tmem_st32(lane_addr + kTokT * (t & 1) + 32 * part, pp);
      }
      tmem_wait_st();
      tc_fence_before();
      if (!dead) mbar_arrive(pready);
    }
    if (!dead && !mbar_wait_bounded(pvdone + 8 * ((ntile - 1) & 1), static_cast<uint32_t>(((ntile - 1) >> 1) & 1),
                                    kWaitT))
      dead = true;
    tc_fence_after();
    if (dead && lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);

    // o'/l of this part of the row (the row sum gathers the four parts' in shared memory).
    lsum[part * kRowsT + row] = l;
    float o[32];
    {
      uint32_t r[32];
      tmem_ld32(lane_addr + kColO + 32 * part, r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; e++) o[e] = __uint_as_float(r[e]);
    }
    asm volatile("bar.sync %0, 128;" ::"r"(1 + quarter) : "memory");
    float lt = 0.0f;
#pragma unroll
    for (int q2 = 0; q2 < 4; q2++) lt += lsum[q2 * kRowsT + row];
    const float il = lt > 0.0f ? __frcp_rn(lt) : 0.0f;
#pragma unroll
    for (int e = 0; e < 32; e++) o[e] *= il;
    // Inverse block Hadamard: stages h = 1..16 inside the part, h = 32 and 64 across parts
    // (through the K buffers, free once the last QK^T has completed; channel-major so a
    // warp's accesses are contiguous).
    const int block = p.hadamard_block;
#pragma unroll
    for (int hh = 1; hh < 32; hh *= 2) {
      if (hh < block) {
#pragma unroll
        for (int i = 0; i < 32; i++)
          if (!(i & hh)) {
            const float a = o[i], d = o[i + hh];
            o[i] = a + d;
            o[i + hh] = a - d;
          }
      }
    }
    float* xch = reinterpret_cast<float*>(smem + kQh);  // [part][32 channels][128 rows]
#pragma unroll
    for (int st = 0; st < 2; st++) {
      const int hp = 1 << st;  // partner part: channels differ by 32 hp
      if ((32 << st) < block) {
#pragma unroll
        for (int e = 0; e < 32; e++) xch[(part * 32 + e) * kRowsT + row] = o[e];
        asm volatile("bar.sync %0, 128;" ::"r"(1 + quarter) : "memory");
#pragma unroll
        for (int e = 0; e < 32; e++) {
          const float other = xch[((part ^ hp) * 32 + e) * kRowsT + row];
          o[e] = (part & hp) ? other - o[e] : o[e] + other;
        }
        asm volatile("bar.sync %0, 128;" ::"r"(1 + quarter) : "memory");
      }
    }
    if (row_valid && !dead) {
      __half* orow = p.out + ((static_cast<size_t>(cq0) + ti_row) * p.num_kv_heads * G + h * G + row % G) * kD +
                     32 * part;
#pragma unroll
      for (int c8 = 0; c8 < 4; c8++) {
        const float* v = o + 8 * c8;
        *reinterpret_cast<uint4*>(orow + 8 * c8) = make_uint4(
            pack_half2(__float2half_rn(v[0] * p.cb), __float2half_rn(v[1] * p.cb)),
            pack_half2(__float2half_rn(v[2] * p.cb), __float2half_rn(v[3] * p.cb)),
            pack_half2(__float2half_rn(v[4] * p.cb), __float2half_rn(v[5] * p.cb)),
            pack_half2(__float2half_rn(v[6] * p.cb), __float2half_rn(v[7] * p.cb)));
      }
    }
  } else if (w < kExpWarp0 + kExpWarps) {
    // -------------------------------------------------------------- expansion warps --
    // Items: tokens ej and ej + 64 of the tile, channels 64 ehf..64 ehf + 63, for K and V.
    const int eid = tid - kExpWarp0 * 32, ej0 = eid >> 1, ehf = eid & 1;
    for (int t = 0; t <= ntile; t++) {
      if (t < ntile) {
        // K of tile t into K buffer t & 1 (free once the softmax of tile t - 2 has read S and
        // the K scales, which also means QK^T of t - 2 has completed).
        const int slot = t % F::kStages;
        if (!dead && !mbar_wait_bounded(full_s + 8 * slot, static_cast<uint32_t>((t / F::kStages) & 1), kWaitT))
          dead = true;
        if (t >= 2 && !dead &&
            !mbar_wait_bounded(sfree + 8 * (t & 1), static_cast<uint32_t>(((t - 2) >> 1) & 1), kWaitT))
          dead = true;
        if (!dead) {
#pragma unroll
          for (int it = 0; it < 2; it++) {
            const int ej = ej0 + 64 * it;
            const uint8_t* pg = smem + kRing + slot * F::kSlot + (ej / SEFF) * (SEFF * F::kRowB);
            const int jr = ej % SEFF;
            if constexpr (FP4) {
              const bool live = t * kTokT + ej < L;
              expand_fp4_half<SEFF>(pg, jr, 0, ehf, live, smem + kKs + (t & 1) * kKsBuf + ehf * (kTokT * 128), ej);
              if (ehf == 0) s_kb[(t & 1) * kTokT + ej] = live ? 1.0f : 0.0f;
              continue;
            }
            const uint4* src = reinterpret_cast<const uint4*>(pg + jr * 64 + 32 * ehf);
            const uint4 c0 = src[0], c1 = src[1];
            const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint8_t* kb = smem + kKs + (t & 1) * kKsBuf + ehf * (kTokT * 128);
#pragma unroll
            for (int ch = 0; ch < 8; ch++)  // 16-byte chunk ch = channels 64 ehf + 8 ch .. + 7
              *reinterpret_cast<uint4*>(kb + sw_off(ej, ch)) =
                  make_uint4(codes_f16x2(cw[ch], 0), codes_f16x2(cw[ch], 1), codes_f16x2(cw[ch], 2),
                             codes_f16x2(cw[ch], 3));
            if (ehf == 0) {
              const bool live = t * kTokT + ej < L;
              const __half sk = reinterpret_cast<const __half*>(pg + SEFF * 128)[jr];
              s_kb[(t & 1) * kTokT + ej] = live ? __half2float(sk) : 0.0f;
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(kready + 8 * (t & 1));
        }
      }
      if (t >= 1) {
        // V of tile u = t - 1 into V buffer u & 1 (free once PV of u - 2 has completed,
        // which also means the softmax of u - 2 has read its V scales).
        const int u = t - 1, slot = u % F::kStages;
        if (u >= 2 && !dead &&
            !mbar_wait_bounded(pvdone + 8 * (u & 1), static_cast<uint32_t>(((u - 2) >> 1) & 1), kWaitT))
          dead = true;
        if (FP4 && !dead) {
#pragma unroll
          for (int it = 0; it < 2; it++) {
            const int ej = ej0 + 64 * it;
            const uint8_t* pg = smem + kRing + slot * F::kSlot + (ej / SEFF) * (SEFF * F::kRowB);
            const bool live = u * kTokT + ej < L;
            expand_fp4_half<SEFF>(pg, ej % SEFF, 1, ehf, live, smem + kVs + (u & 1) * kVsBuf + ehf * (kTokT * 128),
                                  ej);
            if (ehf == 0) s_vb[(u & 1) * kTokT + ej] = live ? 1.0f : 0.0f;
          }
          // The raw slot of tile u is fully read: the producer may refill it.
          mbar_arrive(empty_s + 8 * slot);
          fence_proxy_async_smem();
          mbar_arrive(vready + 8 * (u & 1));
        }
        if (!FP4 && !dead) {
          uint32_t cw[2][8];
          float vs[2] = {0.0f, 0.0f};
#pragma unroll
          for (int it = 0; it < 2; it++) {
            const int ej = ej0 + 64 * it;
            const uint8_t* pg = smem + kRing + slot * F::kSlot + (ej / SEFF) * (SEFF * F::kRowB);
            const int jr = ej % SEFF;
            const uint4* src = reinterpret_cast<const uint4*>(pg + SEFF * 64 + jr * 64 + 32 * ehf);
            const uint4 c0 = src[0], c1 = src[1];
            cw[it][0] = c0.x; cw[it][1] = c0.y; cw[it][2] = c0.z; cw[it][3] = c0.w;
            cw[it][4] = c1.x; cw[it][5] = c1.y; cw[it][6] = c1.z; cw[it][7] = c1.w;
            if (ehf == 0 && u * kTokT + ej < L)
              vs[it] = __half2float(reinterpret_cast<const __half*>(pg + SEFF * 130)[jr]);
          }
          // The raw slot of tile u is fully read: the producer may refill it.
          mbar_arrive(empty_s + 8 * slot);
#pragma unroll
          for (int it = 0; it < 2; it++) {
            const int ej = ej0 + 64 * it;
            uint8_t* vb = smem + kVs + (u & 1) * kVsBuf + ehf * (kTokT * 128);
#pragma unroll
            for (int ch = 0; ch < 8; ch++) {
              const uint32_t wv = cw[it][ch], wvh = wv >> 4;
              *reinterpret_cast<uint4*>(vb + sw_off(ej, ch)) =
                  make_uint4(codes_bf16x2(wv, wvh, 0), codes_bf16x2(wv, wvh, 1), codes_bf16x2(wv, wvh, 2),
                             codes_bf16x2(wv, wvh, 3));
            }
            if (ehf == 0) s_vb[(u & 1) * kTokT + ej] = vs[it];
          }
          fence_proxy_async_smem();
          mbar_arrive(vready + 8 * (u & 1));
        }
      }
    }
    if (dead && lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);
  } else if (w == kMmaWarp) {
    // ------------------------------------------------------------------- MMA warp --
    // One elected lane issues; the whole warp walks the waits so it stays converged.
    const uint64_t dk0 = smem_desc_sw128(sbase + kKs, 16, 1024);
    const uint64_t dv0 = smem_desc_sw128(sbase + kVs, kTokT * 128, 1024);
    uint32_t last_bar = 0, last_par = 0;  // the latest commit (it covers every earlier MMA)
    for (int t = 0; t <= ntile; t++) {
      if (t < ntile) {
        // S[t & 1] = q~hi . K + q~lo . K over 8 k-steps of 16 channels.
        const uint32_t par = static_cast<uint32_t>((t >> 1) & 1);
        if (!dead && !mbar_wait_bounded(kready + 8 * (t & 1), par, kWaitT)) dead = true;
        if (t >= 2 && !dead &&
            !mbar_wait_bounded(sfree + 8 * (t & 1), static_cast<uint32_t>(((t - 2) >> 1) & 1), kWaitT))
          dead = true;
        tc_fence_after();
        if (!dead && lane == 0) {
          const uint64_t dk = dk0 + static_cast<uint64_t>(((t & 1) * kKsBuf) >> 4);
#pragma unroll
          for (int s = 0; s < 8; s++) {  // k-step s: channels 16 s.., q~ columns 8 s..
            const uint64_t ko = static_cast<uint64_t>(((s >> 2) * (kTokT * 128u) + (s & 3) * 32u) >> 4);
            tc_mma_f16_ts(tmem + kTokT * (t & 1), tmem + kColQh + 8 * s, dk + ko, kIdescQK, s > 0);
            tc_mma_f16_ts(tmem + kTokT * (t & 1), tmem + kColQl + 8 * s, dk + ko, kIdescQK, 1u);
          }
          tc_commit(sfull + 8 * (t & 1));
        }
        if (!dead) { last_bar = sfull + 8 * (t & 1); last_par = par; }
        __syncwarp();
      }
      if (t >= 1) {
        // O (+)= P'hi . V + P'lo . V over 4 k-steps of 16 tokens, tile u = t - 1.
        const int u = t - 1;
        const uint32_t par = static_cast<uint32_t>((u >> 1) & 1);
        if (!dead && !mbar_wait_bounded(pready, static_cast<uint32_t>(u & 1), kWaitT)) dead = true;
        if (!dead && !mbar_wait_bounded(vready + 8 * (u & 1), par, kWaitT)) dead = true;
        tc_fence_after();
        if (!dead && lane == 0) {
          const uint64_t dv = dv0 + static_cast<uint64_t>(((u & 1) * kVsBuf) >> 4);
#pragma unroll
          for (int s = 0; s < 8; s++) {  // k-step s: tokens 16 s.., P' of half s / 4, chunk (s / 2) % 2
            const uint64_t vd = dv + static_cast<uint64_t>((2048u * s) >> 4);
            const uint32_t pa = tmem + kTokT * (u & 1) + 32 * (s >> 1) + 8 * (s & 1);
            constexpr uint32_t idesc = FP4 ? kIdescPVh : kIdescPV;
            tc_mma_f16_ts(tmem + kColO, pa, vd, idesc, (u > 0 || s > 0) ? 1u : 0u);
            tc_mma_f16_ts(tmem + kColO, pa + 16, vd, idesc, 1u);
          }
          tc_commit(pvdone + 8 * (u & 1));
        }
        if (!dead) { last_bar = pvdone + 8 * (u & 1); last_par = par; }
        __syncwarp();
      }
    }
    if (dead) {
      if (lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);
      // Let the MMAs issued so far finish (bounded) before tensor memory is released.
      if (lane == 0 && last_bar) mbar_wait_bounded(last_bar, last_par, kWaitT);
    }
  } else if (w == kProdWarp) {
    // ----------------------------------------------------------------- producer warp --
    // Tile t refills slot t % kStages once the expansion has released tile t - kStages; its
    // page ids are read one tile ahead, so the read overlaps that wait.
    int issued = min(F::kStages, ntile);
    int pid_next = F::kStages < ntile ? tile_page<SEFF, FP4>(F::kStages, b, L, lane, p) : 0;
    for (int t = F::kStages; t < ntile && !dead; t++) {
      const int pid_after = t + 1 < ntile ? tile_page<SEFF, FP4>(t + 1, b, L, lane, p) : 0;
      const int slot = t % F::kStages;
      // Lane 0 waits and tells the others, so the warp stays converged for the copies.
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(empty_s + 8 * slot, static_cast<uint32_t>((t / F::kStages - 1) & 1), kWaitT);
      if (!__shfl_sync(kFullT, ok, 0)) {
        dead = true;
        break;
      }
      issue_tile_pages<SEFF, FP4>(t, h, L, pid_next, sbase + kRing + slot * F::kSlot, full_s + 8 * slot, lane, pol, p);
      issued++;
      pid_next = pid_after;
    }
    if (dead && lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);
    // Before shared memory is released, the last copies into each slot must have landed
    // (bounded; earlier ones were consumed by the expansion before their slot was reused).
    if (lane == 0)
      for (int j = max(0, issued - F::kStages); j < issued; j++)
        mbar_wait_bounded(full_s + 8 * (j % F::kStages), static_cast<uint32_t>((j / F::kStages) & 1), kWaitT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w == 0) tmem_dealloc(tmem, kTmemCols);
}

template <int G, bool FP4>
void* prefill_tc_ptr(int seff) {
  if (seff == 16) return reinterpret_cast<void*>(&prefill_tc_kernel<G, 16, FP4>);
  if (seff == 32) return reinterpret_cast<void*>(&prefill_tc_kernel<G, 32, FP4>);
  if (seff == 64) return reinterpret_cast<void*>(&prefill_tc_kernel<G, 64, FP4>);
  if (seff == 128) return reinterpret_cast<void*>(&prefill_tc_kernel<G, 128, FP4>);
  return nullptr;
}

template <bool FP4>
void* pick_prefill_tc(int group, int seff) {
  switch (group) {
    case 1: return prefill_tc_ptr<1, FP4>(seff);
    case 2: return prefill_tc_ptr<2, FP4>(seff);
    case 4: return prefill_tc_ptr<4, FP4>(seff);
    case 8: return prefill_tc_ptr<8, FP4>(seff);
    default: return nullptr;
  }
}

size_t prefill_tc_smem(int max_batch, bool fp4) {
  const int preq = fp4 ? TcFmt<true>::kPreq : TcFmt<false>::kPreq;
  return static_cast<size_t>(preq) + static_cast<size_t>(max_batch + 1) * sizeof(int32_t) + 1024;
}

}  // namespace

int launch_prefill_tc(const PrefillParams& p, int total_q, cudaStream_t stream) {
  const int seff = p.page_size < kTokT ? p.page_size : kTokT;
  void* fn = p.fp4 ? pick_prefill_tc<true>(p.group, seff) : pick_prefill_tc<false>(p.group, seff);
  if (!fn) return -1;
  if (p.batch == 0 || total_q == 0) return 0;
  const int QB = kRowsT / p.group;
  const long long blocks = (static_cast<long long>(total_q) + QB - 1) / QB + p.batch;
  const long long grid = blocks * p.num_kv_heads;
  if (grid > 0x7fffffffLL) return -1;
  const size_t smem = prefill_tc_smem(p.batch, p.fp4 != 0);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(prefill_tc_smem(4096, p.fp4 != 0))) != cudaSuccess)
    return -2;
  PrefillParams q = p;
  q.total_q = total_q;
  void* args[] = {&q};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreadsT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) return -2;
  return 0;
}

}  // namespace kvq

// prefill_kernel.cu -- causal chunked-prefill attention over the rotated-INT4 paged KV
// cache, for sm_100a.
//
// Method: "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化"
// (youngju.dev): section "KVキャッシュこそが本当のボトルネックである理由" (attention runs
// over the paged cache in serving engines) and "回転のトリック — ブロック対角アダマール"
// (the orthonormal rotation keeps q.k, so attention runs in the rotated domain and the
// output is rotated back).  A chunk of C prompt tokens of a sequence, already appended,
// attends the cache causally: query i of the chunk (position L - C + i) sees positions
// 0..L - C + i.
//
// Work decomposition.  A CTA (4 warps) takes 64 query rows of one (sequence, KV head):
// QB = 64 / G consecutive chunk tokens times the G query heads of the KV head; warp w owns
// rows 16w..16w+15 end to end (its own online softmax, no cross-warp merge).  The CTA
// streams the causal KV range of its rows in tiles of 32 tokens through one shared ring of
// 3 slots filled by bulk copies (cp.async.bulk, issued by warp 0; every warp releases a
// slot by one arrival on the slot's "empty" barrier).  Per tile and warp:
//   QK^T  int8 mma m16n8k32, A = q' cut into three int8 slices (as in decode; read from
//         shared memory with ldmatrix), B = K codes as int8 (nibble moved to the byte's
//         top), 4 n-tiles of 8 tokens; scores in the log2 domain with the K scale and the
//         row's slice scale; causal mask on positions.
//   softmax  online, per row; the row sum stays lane-partial until the end.
//   PV    fp16 mma m16n8k16, A = P' = p * s_v as fp16 hi + lo (the score accumulators are
//         the A fragments, no shuffles), B = V codes as exact fp16 (byte gather + magic
//         conversion), 16 n-tiles of 8 channels.
// The end: o'/l, the inverse block Hadamard across a row's channels (bits 1-2 of the
// channel across lanes, the others in registers), times c_b, fp16 store.
//
// NVFP4 cache (template argument FP4; "BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号"
// (sns.style): E2M1 codes with an E4M3 scale per 16 channels, 144-byte token rows): K is
// dequantised exactly to fp16 once per CTA and tile into a second swizzled stage, like V;
// QK^T runs as fp16 mma m16n8k16 with q' carried as fp16 hi + lo parts (both accumulate into
// one accumulator), B fragments read with ldmatrix; P' = p.  Scales of tokens past the
// sequence's end are taken as 0 in both stages (their slot bytes are stale).
#include <cuda_fp16.h>
#include <math_constants.h>
#include <stdint.h>

#include "../../include/kvq.h"
#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kD = 128;
constexpr int kRows = 64;        // query rows per CTA
constexpr int kWarpsP = 4;
constexpr int kThreadsP = 128;
constexpr int kStagesP = 3;
// Token row of a (page, head) block (INT4: codes + 2 fp16 scales; NVFP4: codes + 2 x 8 E4M3
// scales) and the ring slot of one 32-token tile.
constexpr int row_bytes_p(bool fp4) { return fp4 ? kD + kD / 8 : kD + 4; }
constexpr int slot_bytes_p(bool fp4) { return kTileTokens * row_bytes_p(fp4); }
constexpr unsigned kFullMask = 0xffffffffu;
constexpr float kMagicP = 12582912.0f;  // 1.5 * 2^23
constexpr uint64_t kWaitNs = 2000000000ull;

__device__ __forceinline__ void split_hi_lo_p(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(p0, p1);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(p0 - f.x, p1 - f.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Byte offset of token tau (0..31) of a ring slot: the slot holds pages of SEFF token
// slots in the pool's block layout [K codes][V codes][K scales][V scales].
template <int SEFF, bool FP4>
__device__ __forceinline__ int tok_base(int tau) {
  return (tau / SEFF) * (SEFF * row_bytes_p(FP4));
}

// Issue the bulk copies of tile t (tokens 32t..) of sequence b, KV head h into a slot
// (warp 0 calls; lane j < pages-needed copies page j).
template <int SEFF, bool FP4>
__device__ __forceinline__ void issue_tile(int t, int b, int h, int L, uint32_t slot, uint32_t bar,
                                           int lane, uint64_t pol, const PrefillParams& p) {
  const int S = p.page_size, sh = p.page_shift;
  const uint32_t blk_bytes = static_cast<uint32_t>(S) * row_bytes_p(FP4);
  const int t0 = t * kTileTokens;
  const int t1 = min(t0 + kTileTokens, L);  // > t0
  if (SEFF < kTileTokens || S == kTileTokens) {
    const int npg = ((t1 - 1) >> sh) - (t0 >> sh) + 1;
    int pid = 0;
    bool bad = false;
    if (lane < npg) {
      pid = __ldg(p.page_table + static_cast<size_t>(b) * p.max_pages_per_seq + (t0 >> sh) + lane);
      bad = pid < 0 || pid >= p.num_pages;
      if (bad) pid = 0;
    }
    if (__any_sync(kFullMask, bad) && lane == 0) atomicOr(p.status, KVQ_DEV_BAD_PAGE_BIT);
    if (lane == 0) mbar_arrive_expect_tx(bar, npg * blk_bytes);
    __syncwarp();
    if (lane < npg)
      bulk_copy_g2s(slot + lane * blk_bytes,
                    p.pool_layer + (static_cast<size_t>(pid) * p.num_kv_heads + h) * blk_bytes,
                    blk_bytes, bar, pol);
  } else {
    int pid = __ldg(p.page_table + static_cast<size_t>(b) * p.max_pages_per_seq + (t0 >> sh));
    const bool bad = pid < 0 || pid >= p.num_pages;
    if (bad) pid = 0;
    if (bad && lane == 0) atomicOr(p.status, KVQ_DEV_BAD_PAGE_BIT);
    const size_t o = static_cast<size_t>(t0 & (S - 1));
    const uint8_t* blk = p.pool_layer + (static_cast<size_t>(pid) * p.num_kv_heads + h) * blk_bytes;
    const uint8_t* src = blk + o * 64;
    uint32_t dst = slot, bytes = 2048;
    if constexpr (FP4) {  // scales: 8 E4M3 bytes per token row
      if (lane == 1) { src = blk + static_cast<size_t>(S) * 64 + o * 64; dst = slot + 2048; }
      if (lane == 2) { src = blk + static_cast<size_t>(S) * 128 + o * 8; dst = slot + 4096; bytes = 256; }
      if (lane == 3) { src = blk + static_cast<size_t>(S) * 136 + o * 8; dst = slot + 4352; bytes = 256; }
    } else {
      if (lane == 1) { src = blk + static_cast<size_t>(S) * 64 + o * 64; dst = slot + 2048; }
      if (lane == 2) { src = blk + static_cast<size_t>(S) * 128 + o * 2; dst = slot + 4096; bytes = 64; }
      if (lane == 3) { src = blk + static_cast<size_t>(S) * 130 + o * 2; dst = slot + 4160; bytes = 64; }
    }
    if (lane == 0) mbar_arrive_expect_tx(bar, slot_bytes_p(FP4));
    __syncwarp();
    if (lane < 4) bulk_copy_g2s(dst, src, bytes, bar, pol);
  }
}

// Rotate one q row (lane: channels 4L..4L+3; the fixed butterfly, then x c_b x q_scale),
// cut it into three int8 slices q' = M/64 (q1 + q2/128 + q3/16384), M the power of two >=
// max |q'|, and store the slices in A-fragment order: qs[s][jj][row][kappa] with, inside
// k-step jj, kappa = 4c + e <-> channel 32c + 8jj + 2e and kappa = 16 + 4c + e <-> channel
// 32c + 8jj + 2e + 1.  The two 16-byte halves of a 32-byte row swap places on rows with
// bit 2 set, so that ldmatrix's 8 rows fall in distinct banks.  Returns M / 1024 (the score scale of the row; K codes enter the MMA
// times 16).
__device__ __forceinline__ float prep_q_row(const __half* qrow, bool valid, uint8_t* qs, int row,
                                            int lane, const PrefillParams& p) {
  float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (valid) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qrow) + lane);
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    x[0] = lo.x; x[1] = lo.y; x[2] = hi.x; x[3] = hi.y;
  }
  if (p.hadamard_block > 1) {
    const float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
    x[0] = a0 + a2; x[2] = a0 - a2; x[1] = a1 + a3; x[3] = a1 - a3;
#pragma unroll
    for (int st = 0; st < 5; st++) {
      if ((4 << st) < p.hadamard_block) {
        const float sgn = ((lane >> st) & 1) ? -1.0f : 1.0f;
#pragma unroll
        for (int e = 0; e < 4; e++) x[e] = __fmaf_rn(x[e], sgn, __shfl_xor_sync(kFullMask, x[e], 1 << st));
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
  for (int d = 1; d < 32; d *= 2) amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, d));
  float M = 1.0f;
  if (amax > 1e-30f) {
    const uint32_t bits = __float_as_uint(amax);
    M = (bits & 0x7FFFFFu) ? __uint_as_float((bits & 0x7F800000u) + 0x00800000u) : amax;
  }
  const float inv = 64.0f / M;
  uint32_t ms[3][4];
#pragma unroll
  for (int e = 0; e < 4; e++) {
    const float t = x[e] * inv;
    const float m1 = t + kMagicP;
    const float r1 = (t - (m1 - kMagicP)) * 128.0f;
    const float m2 = r1 + kMagicP;
    const float r2 = (r1 - (m2 - kMagicP)) * 128.0f;
    const float m3 = r2 + kMagicP;
    ms[0][e] = __float_as_uint(m1);
    ms[1][e] = __float_as_uint(m2);
    ms[2][e] = __float_as_uint(m3);
  }
  // Channels 4L + i: c = L/8, jj = (L%8)/2, e = 2(L%2) + i/2, odd = i%2.
  const int c = lane >> 3, jj = (lane & 7) >> 1, e0 = 2 * (lane & 1);
#pragma unroll
  for (int s = 0; s < 3; s++) {
    uint8_t* r = qs + ((s * 4 + jj) * kRows + row) * 32;
    const int sw = ((row >> 2) & 1) * 16;  // swizzle of the 16-byte halves
    const uint16_t ev = static_cast<uint16_t>((ms[s][0] & 0xFFu) | ((ms[s][2] & 0xFFu) << 8));
    const uint16_t od = static_cast<uint16_t>((ms[s][1] & 0xFFu) | ((ms[s][3] & 0xFFu) << 8));
    *reinterpret_cast<uint16_t*>(r + (0 ^ sw) + 4 * c + e0) = ev;
    *reinterpret_cast<uint16_t*>(r + (16 ^ sw) + 4 * c + e0) = od;
  }
  return M * (1.0f / 1024.0f);
}

// NVFP4 path: the same rotated, scaled row normalised to q~ = q' * 2^14 / M and stored as
// fp16 hi + lo parts in A-fragment order: qs[part][kk][row][16 channels], k-step kk =
// channels 16kk..16kk+15 in order, the same 16-byte swizzle as the int8 slices.  Returns
// M / 2^14 (the score scale of the row).
__device__ __forceinline__ float prep_q_row4(const __half* qrow, bool valid, uint8_t* qs, int row,
                                             int lane, const PrefillParams& p) {
  float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (valid) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qrow) + lane);
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    x[0] = lo.x; x[1] = lo.y; x[2] = hi.x; x[3] = hi.y;
  }
  if (p.hadamard_block > 1) {
    const float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
    x[0] = a0 + a2; x[2] = a0 - a2; x[1] = a1 + a3; x[3] = a1 - a3;
#pragma unroll
    for (int st = 0; st < 5; st++) {
      if ((4 << st) < p.hadamard_block) {
        const float sgn = ((lane >> st) & 1) ? -1.0f : 1.0f;
#pragma unroll
        for (int e = 0; e < 4; e++) x[e] = __fmaf_rn(x[e], sgn, __shfl_xor_sync(kFullMask, x[e], 1 << st));
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
  for (int d = 1; d < 32; d *= 2) amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, d));
  float M = 1.0f;
  if (amax > 1e-30f) {
    const uint32_t bits = __float_as_uint(amax);
    M = (bits & 0x7FFFFFu) ? __uint_as_float((bits & 0x7F800000u) + 0x00800000u) : amax;
  }
  const float inv = 16384.0f / M;  // exact: powers of two
  __half hv[4], lv[4];
#pragma unroll
  for (int e = 0; e < 4; e++) {
    const float t = x[e] * inv;
    hv[e] = __float2half_rn(t);
    lv[e] = __float2half_rn(t - __half2float(hv[e]));
  }
  // Channels 4L..4L+3: k-step L/4, bytes 8(L%4).. of the 32-byte row, halves swizzled.
  const int kk = lane >> 2;
  const int off = (8 * (lane & 3)) ^ (((row >> 2) & 1) * 16);
  const uint2 wh = make_uint2(pack_half2(hv[0], hv[1]), pack_half2(hv[2], hv[3]));
  const uint2 wl = make_uint2(pack_half2(lv[0], lv[1]), pack_half2(lv[2], lv[3]));
  *reinterpret_cast<uint2*>(qs + ((0 * 8 + kk) * kRows + row) * 32 + off) = wh;
  *reinterpret_cast<uint2*>(qs + ((1 * 8 + kk) * kRows + row) * 32 + off) = wl;
  return M * (1.0f / 16384.0f);
}

// One byte of two E2M1 codes (low nibble first) -> fp16x2, exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2_p(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
      : "=r"(r)
      : "r"(byte));
  return r;
}

// Two E4M3 bytes (low 16 bits, low byte first) -> fp16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_p(uint32_t b) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(b)));
  return h;
}

__device__ __forceinline__ uint32_t hmul2_p(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// NVFP4 stage: token tau's 32 channels 32part..32part+31 of K (kv = 0) or V (kv = 1),
// dequantised to fp16 (E2M1 value x E4M3 scale, exact) into the swizzled [token][channel]
// stage; scale 0 for a token past the sequence's end.
template <int SEFF>
__device__ __forceinline__ void stage_fp4(const uint8_t* base, int tau, int part, int kv, bool live,
                                          uint8_t* stage) {
  const uint8_t* row = base + tok_base<SEFF, true>(tau);
  const uint4 cw = *reinterpret_cast<const uint4*>(row + kv * SEFF * 64 + (tau % SEFF) * 64 + 16 * part);
  const uint32_t sb = live ? *reinterpret_cast<const uint16_t*>(row + SEFF * 128 + kv * SEFF * 8 +
                                                                (tau % SEFF) * 8 + 2 * part)
                           : 0u;
  const uint32_t s2 = e4m3x2_to_f16x2_p(sb);
  const uint32_t sdup[2] = {prmt(s2, s2, 0x1010u), prmt(s2, s2, 0x3232u)};  // blocks 2part, +1
  const uint32_t wds[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int i = 0; i < 4; i++) {  // 16-byte chunk 4part + i = channels 8(4part + i) ..
    uint32_t hv[4];
#pragma unroll
    for (int k = 0; k < 4; k++) hv[k] = hmul2_p(e2m1x2_to_f16x2_p(wds[i] >> (8 * k)), sdup[i >> 1]);
    const int chunk = (4 * part + i) ^ (tau & 7);
    *reinterpret_cast<uint4*>(stage + tau * 256 + chunk * 16) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
  }
}

template <int G, int SEFF, bool FP4>
__global__ void __launch_bounds__(kThreadsP, 3) prefill_kernel(PrefillParams p) {
  constexpr int QB = kRows / G;  // chunk tokens per CTA
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  constexpr int kSlotP = slot_bytes_p(FP4);
  constexpr int kQsBytes = FP4 ? 2 * 8 * kRows * 32 : 3 * 4 * kRows * 32;
  uint8_t* ring = smem;                                        // [3][slot]
  uint8_t* qs = ring + kStagesP * kSlotP;                      // int8 slices or fp16 hi/lo
  float* sfr = reinterpret_cast<float*>(qs + kQsBytes);        // [64] row scales
  uint8_t* vst = reinterpret_cast<uint8_t*>(sfr + kRows);      // [2][32 tokens][256 B] fp16 V
  uint8_t* kst = vst + 2 * kTileTokens * 256;                  // NVFP4: [2][32][256] fp16 K
  uint64_t* bars = reinterpret_cast<uint64_t*>(kst + (FP4 ? 2 * kTileTokens * 256 : 0));  // full[3], empty[3]
  int32_t* preq = reinterpret_cast<int32_t*>(bars + 2 * kStagesP);  // [batch + 1]
  __shared__ int warp_sum[kWarpsP];
  __shared__ int running;

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  // Before griddep_wait only cu_q, seq_lens and the page table are read (inputs of this
  // call); q, the pool and out are touched after it.
  griddep_launch_dependents();
  const uint32_t full_s = smem_addr(bars), empty_s = smem_addr(bars + kStagesP);
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStagesP; s++) {
      mbar_init(full_s + 8 * s, 1);
      mbar_init(empty_s + 8 * s, kWarpsP);
    }
    fence_mbar_init();
    running = 0;
  }
  __syncthreads();

  // Query blocks per sequence -> exclusive prefix preq[0..batch].
  for (int base = 0; base < p.batch; base += kThreadsP) {
    const int i = base + tid;
    int n = 0;
    if (i < p.batch) {
      const int C = __ldg(p.cu_q + i + 1) - __ldg(p.cu_q + i);
      n = C > 0 ? (C + QB - 1) / QB : 0;
    }
    int incl = n;
#pragma unroll
    for (int d = 1; d < 32; d *= 2) {
      const int y = __shfl_up_sync(kFullMask, incl, d);
      if (lane >= d) incl += y;
    }
    if (lane == 31) warp_sum[w] = incl;
    __syncthreads();
    int before = running;
    for (int w2 = 0; w2 < w; w2++) before += warp_sum[w2];
    if (i < p.batch) preq[i] = before + incl - n;
    __syncthreads();
    if (tid == kThreadsP - 1) running = before + incl;
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
  int L = __ldg(p.seq_lens + b);
  if (L > cap || C > L || cq0 < 0 || cq0 + C > p.total_q) {
    if (tid == 0) atomicOr(p.status, KVQ_DEV_BAD_POS_BIT);
    return;
  }
  const int tok_first = qb * QB;                       // first chunk token of the CTA
  const int tok_last = min(C, tok_first + QB) - 1;     // last valid one
  const int pos_last = L - C + tok_last;
  const int ntile = pos_last / kTileTokens + 1;
  const uint64_t pol = l2_policy_evict_first();

  griddep_wait();

  // The first kStagesP tiles (warp 0), then every warp prepares its 16 q rows.
  int issued = 0, done0 = 0;  // warp 0: tiles issued / tiles whose copy it waited for
  if (w == 0)
    for (; issued < kStagesP && issued < ntile; issued++)
      issue_tile<SEFF, FP4>(issued, b, h, L, smem_addr(ring) + issued * kSlotP,
                            full_s + 8 * issued, lane, pol, p);
  for (int rr = 0; rr < 16; rr++) {
    const int row = 16 * w + rr;
    const int ti = tok_first + row / G, gq = row % G;
    const bool valid = ti < C;
    const __half* qrow = p.q + ((static_cast<size_t>(cq0) + (valid ? ti : 0)) * p.num_kv_heads * G +
                                h * G + gq) * kD;
    const float sf = FP4 ? prep_q_row4(qrow, valid, qs, row, lane, p)
                         : prep_q_row(qrow, valid, qs, row, lane, p);
    if (lane == 0) sfr[row] = sf;
  }
  __syncwarp();

  // This lane's rows: g and g + 8 of the warp's 16.
  const int r0 = 16 * w + g, r1 = r0 + 8;
  const float sf0 = sfr[r0], sf1 = sfr[r1];
  const int pos0 = L - C + tok_first + r0 / G, pos1 = L - C + tok_first + r1 / G;
  const int pos_min = L - C + tok_first + (16 * w) / G;  // the warp's first row's position
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.0f, l1 = 0.0f;
  const uint32_t qs_s = smem_addr(qs);
  // ldmatrix row address of this lane inside a [64][32] slice block: matrix L/8.
  const int lm = lane >> 3, lr = lane & 7;
  const int a_row = 16 * w + lr + (lm & 1) * 8;
  const uint32_t a_off = static_cast<uint32_t>(a_row * 32 + (((lm >> 1) ^ ((a_row >> 2) & 1)) * 16));
  bool dead = false;

  for (int t = 0; t < ntile; t++) {
    const int slot = t % kStagesP;
    const uint32_t par = static_cast<uint32_t>((t / kStagesP) & 1);
    if (!dead) {
      if (mbar_wait_bounded(full_s + 8 * slot, par, kWaitNs)) done0++;
      else dead = true;
    }
    const uint8_t* base = ring + slot * kSlotP;
    // The tile's V codes as fp16, once per CTA: warp w converts tokens 8w..8w+7 into the
    // stage t % 2 ([token][channel], the 16-byte chunk index XOR (token & 7), so ldmatrix's
    // 8 rows fall in distinct banks).  The barrier below also tells every warp that all
    // warps are done with the stage's previous tile.
    uint8_t* vs = vst + (t & 1) * (kTileTokens * 256);
    uint8_t* ks = kst + (t & 1) * (kTileTokens * 256);  // NVFP4 only
    if (FP4 && !dead) {
      const int tau = 8 * w + (lane >> 2), part = lane & 3;  // channels 32part .. 32part+31
      const bool live = t * kTileTokens + tau < L;
      stage_fp4<SEFF>(base, tau, part, 0, live, ks);
      stage_fp4<SEFF>(base, tau, part, 1, live, vs);
    }
    if (!FP4 && !dead) {
      const int tau = 8 * w + (lane >> 2), part = lane & 3;  // channels 32part .. 32part+31
      const uint4 cw = *reinterpret_cast<const uint4*>(base + tok_base<SEFF, FP4>(tau) + SEFF * 64 +
                                                       (tau % SEFF) * 64 + 16 * part);
      const uint32_t wds[4] = {cw.x, cw.y, cw.z, cw.w};
      uint32_t hv[16];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int k = 0; k < 4; k++) {
          // byte k of word i: channels 32part + 8i + 2k (low nibble), +1 (high nibble)
          uint32_t x = prmt(wds[i], 0u, static_cast<uint32_t>(k) | (static_cast<uint32_t>(k) << 8) | 0x4040u);
          x = lop3_and_xor(x, 0x00F0000Fu, 0x64806408u);
          asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(x) : "r"(x), "r"(0x2C003C00u), "r"(0xD480E408u));
          hv[4 * i + k] = x;
        }
#pragma unroll
      for (int i = 0; i < 4; i++) {  // 16-byte chunk 4part + i = channels 8(4part + i) ..
        const int chunk = (4 * part + i) ^ (tau & 7);
        *reinterpret_cast<uint4*>(vs + tau * 256 + chunk * 16) =
            make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
      }
    }
    __syncthreads();
    if (!dead) {
      float sc[4][4];
      float sk[4][2], sv[4][2];
      if constexpr (FP4) {
        // Scores: fp16 q~ hi and lo parts against the fp16 K stage (k-step kk = channels
        // 16kk..16kk+15; ldmatrix of two n-tiles of 8 tokens at once), one accumulator.
        float acc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; nt++) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < 8; kk++) {
          uint32_t h0, h1, h2, h3, l0_, l1_, l2_, l3_;
          ldsm_x4(qs_s + static_cast<uint32_t>((0 * 8 + kk) * kRows * 32) + a_off, h0, h1, h2, h3);
          ldsm_x4(qs_s + static_cast<uint32_t>((1 * 8 + kk) * kRows * 32) + a_off, l0_, l1_, l2_, l3_);
#pragma unroll
          for (int np = 0; np < 4; np += 2) {
            const int ktok = 8 * (np + (lm >> 1)) + lr;
            const int kch = 2 * kk + (lm & 1);
            uint32_t b0a, b1a, b0b, b1b;
            ldsm_x4(smem_addr(ks) + static_cast<uint32_t>(ktok * 256 + ((kch ^ (ktok & 7)) * 16)),
                    b0a, b1a, b0b, b1b);
            mma_16816(acc[np], h0, h1, h2, h3, b0a, b1a);
            mma_16816(acc[np], l0_, l1_, l2_, l3_, b0a, b1a);
            mma_16816(acc[np + 1], h0, h1, h2, h3, b0b, b1b);
            mma_16816(acc[np + 1], l0_, l1_, l2_, l3_, b0b, b1b);
          }
        }
#pragma unroll
        for (int nt = 0; nt < 4; nt++) {
#pragma unroll
          for (int e = 0; e < 4; e++) sc[nt][e] = acc[nt][e];
          // K scales are inside the stage; V scales inside the V stage (0 past the end).
          const int tpos = t * kTileTokens + 8 * nt + 2 * c;
          sk[nt][0] = sk[nt][1] = 1.0f;
          sv[nt][0] = tpos < L ? 1.0f : 0.0f;
          sv[nt][1] = tpos + 1 < L ? 1.0f : 0.0f;
        }
      } else {
      // K codes of tokens 8nt + g (bytes 16c..16c+15 of the row) and the K/V scales of
      // tokens 8nt + 2c, 8nt + 2c + 1.
      uint4 kr[4];
#pragma unroll
      for (int nt = 0; nt < 4; nt++) {
        const int tau = 8 * nt + g;
        kr[nt] = *reinterpret_cast<const uint4*>(base + tok_base<SEFF, FP4>(tau) + (tau % SEFF) * 64 + 16 * c);
        const int tk = 8 * nt + 2 * c;
        const uint8_t* pb = base + tok_base<SEFF, FP4>(tk);
        const __half2 k2 = *reinterpret_cast<const __half2*>(pb + SEFF * 128 + (tk % SEFF) * 2);
        const __half2 v2 = *reinterpret_cast<const __half2*>(pb + SEFF * 130 + (tk % SEFF) * 2);
        const float2 kf = __half22float2(k2), vf = __half22float2(v2);
        // Slots past the sequence's end hold stale bytes: their V scale must not reach P'.
        const int tpos = t * kTileTokens + tk;
        sk[nt][0] = kf.x; sk[nt][1] = kf.y;
        sv[nt][0] = tpos < L ? vf.x : 0.0f;
        sv[nt][1] = tpos + 1 < L ? vf.y : 0.0f;
      }
      // Scores: three int8 slices.  Slice 2's accumulators are multiplied by 128 and slice
      // 3's MMAs accumulate on top of them, so acc = acc2 * 128 + acc3 exactly (|acc_s| <=
      // 2^20 fits); then s = s1 + acc * 2^-14.
      int acc[4][4];
#pragma unroll
      for (int s = 0; s < 3; s++) {
        if (s < 2) {
#pragma unroll
          for (int nt = 0; nt < 4; nt++) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;
        }
#pragma unroll
        for (int jj = 0; jj < 4; jj++) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(qs_s + static_cast<uint32_t>((s * 4 + jj) * kRows * 32) + a_off, a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < 4; nt++) {
            const uint32_t wv = jj == 0 ? kr[nt].x : jj == 1 ? kr[nt].y : jj == 2 ? kr[nt].z : kr[nt].w;
            mma_16832_s8(acc[nt], a0, a1, a2, a3, (wv << 4) & 0xF0F0F0F0u, wv & 0xF0F0F0F0u);
          }
        }
#pragma unroll
        for (int nt = 0; nt < 4; nt++)
#pragma unroll
          for (int e = 0; e < 4; e++) {
            if (s == 0) sc[nt][e] = static_cast<float>(acc[nt][e]);
            else if (s == 1) acc[nt][e] *= 128;
            else sc[nt][e] += static_cast<float>(acc[nt][e]) * (1.0f / 16384.0f);
          }
      }
      }  // INT4 scores
      // Scale, causal mask (only on tiles reaching past the warp's first row), row maxima.
      float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
      if (t * kTileTokens + kTileTokens - 1 <= pos_min) {
#pragma unroll
        for (int nt = 0; nt < 4; nt++)
#pragma unroll
          for (int e = 0; e < 2; e++) {
            sc[nt][e] *= sf0 * sk[nt][e];
            sc[nt][2 + e] *= sf1 * sk[nt][e];
            mx0 = fmaxf(mx0, sc[nt][e]);
            mx1 = fmaxf(mx1, sc[nt][2 + e]);
          }
      } else {
#pragma unroll
        for (int nt = 0; nt < 4; nt++)
#pragma unroll
          for (int e = 0; e < 2; e++) {
            const int tpos = t * kTileTokens + 8 * nt + 2 * c + e;
            sc[nt][e] = tpos <= pos0 ? sc[nt][e] * (sf0 * sk[nt][e]) : -CUDART_INF_F;
            sc[nt][2 + e] = tpos <= pos1 ? sc[nt][2 + e] * (sf1 * sk[nt][e]) : -CUDART_INF_F;
            mx0 = fmaxf(mx0, sc[nt][e]);
            mx1 = fmaxf(mx1, sc[nt][2 + e]);
          }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      // A row with no visible token yet keeps m = -inf and p = 0.
      const float al0 = mn0 == -CUDART_INF_F ? 1.0f : ex2_approx(m0 - mn0);
      const float al1 = mn1 == -CUDART_INF_F ? 1.0f : ex2_approx(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      float ps0 = 0.0f, ps1 = 0.0f;
#pragma unroll
      for (int nt = 0; nt < 4; nt++)
#pragma unroll
        for (int e = 0; e < 2; e++) {
          sc[nt][e] = mn0 == -CUDART_INF_F ? 0.0f : ex2_approx(sc[nt][e] - mn0);
          sc[nt][2 + e] = mn1 == -CUDART_INF_F ? 0.0f : ex2_approx(sc[nt][2 + e] - mn1);
          ps0 += sc[nt][e];
          ps1 += sc[nt][2 + e];
        }
      l0 = l0 * al0 + ps0;
      l1 = l1 * al1 + ps1;
      if (__any_sync(kFullMask, al0 != 1.0f || al1 != 1.0f)) {
#pragma unroll
        for (int cn = 0; cn < 16; cn++) {
          o[cn][0] *= al0;
          o[cn][1] *= al0;
          o[cn][2] *= al1;
          o[cn][3] *= al1;
        }
      }
      // PV: two k-steps of 16 tokens.
#pragma unroll
      for (int kk = 0; kk < 2; kk++) {
        uint32_t ah[4], al[4];
        split_hi_lo_p(sc[2 * kk][0] * sv[2 * kk][0], sc[2 * kk][1] * sv[2 * kk][1], ah[0], al[0]);
        split_hi_lo_p(sc[2 * kk][2] * sv[2 * kk][0], sc[2 * kk][3] * sv[2 * kk][1], ah[1], al[1]);
        split_hi_lo_p(sc[2 * kk + 1][0] * sv[2 * kk + 1][0], sc[2 * kk + 1][1] * sv[2 * kk + 1][1],
                      ah[2], al[2]);
        split_hi_lo_p(sc[2 * kk + 1][2] * sv[2 * kk + 1][0], sc[2 * kk + 1][3] * sv[2 * kk + 1][1],
                      ah[3], al[3]);
        // B fragments of 2 channel n-tiles per ldmatrix: matrices (tokens 16kk..+7 |
        // 16kk+8..+15) x (n-tile cp | cp + 1), transposed.
#pragma unroll
        for (int cp = 0; cp < 16; cp += 2) {
          const int vtok = 16 * kk + (lm & 1) * 8 + lr;
          const int vch = cp + (lm >> 1);  // 16-byte chunk = channel n-tile
          uint32_t b0a, b1a, b0b, b1b;
          ldsm_x4_trans(smem_addr(vs) + static_cast<uint32_t>(vtok * 256 + ((vch ^ (vtok & 7)) * 16)),
                        b0a, b1a, b0b, b1b);
          mma_16816(o[cp], ah[0], ah[1], ah[2], ah[3], b0a, b1a);
          mma_16816(o[cp], al[0], al[1], al[2], al[3], b0a, b1a);
          mma_16816(o[cp + 1], ah[0], ah[1], ah[2], ah[3], b0b, b1b);
          mma_16816(o[cp + 1], al[0], al[1], al[2], al[3], b0b, b1b);
        }
      }
    }
    // Release the slot; warp 0 refills it with tile t + kStagesP once every warp is done.
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_s + 8 * slot);
    if (w == 0 && !dead && t + kStagesP < ntile) {
      if (!mbar_wait_bounded(empty_s + 8 * slot, par, kWaitNs)) {
        dead = true;
      } else {
        fence_proxy_async_smem();
        issue_tile<SEFF, FP4>(t + kStagesP, b, h, L, smem_addr(ring) + slot * kSlotP,
                         full_s + 8 * slot, lane, pol, p);
        issued++;
      }
    }
  }
  if (dead && lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);

  // Row sums across the 4 lanes of a row; o'/l; inverse rotation; fp16 store.
  l0 += __shfl_xor_sync(kFullMask, l0, 1);
  l0 += __shfl_xor_sync(kFullMask, l0, 2);
  l1 += __shfl_xor_sync(kFullMask, l1, 1);
  l1 += __shfl_xor_sync(kFullMask, l1, 2);
  const float i0 = l0 > 0.0f ? __frcp_rn(l0) : 0.0f, i1 = l1 > 0.0f ? __frcp_rn(l1) : 0.0f;
#pragma unroll
  for (int cn = 0; cn < 16; cn++) {
    o[cn][0] *= i0;
    o[cn][1] *= i0;
    o[cn][2] *= i1;
    o[cn][3] *= i1;
  }
  // Channel 8cn + 2c + e: bit 0 = e (in register pair), bits 1-2 = c (lanes ^1, ^2),
  // bits 3-6 = cn (registers).  Stages h = 1, 2, ..., b/2 in this order.
  const int block = p.hadamard_block;
  if (block > 1) {
#pragma unroll
    for (int cn = 0; cn < 16; cn++) {
      float a = o[cn][0], d = o[cn][1];
      o[cn][0] = a + d; o[cn][1] = a - d;
      a = o[cn][2]; d = o[cn][3];
      o[cn][2] = a + d; o[cn][3] = a - d;
    }
#pragma unroll
    for (int st = 0; st < 2; st++) {
      if ((2 << st) < block) {
        const float sgn = ((c >> st) & 1) ? -1.0f : 1.0f;
#pragma unroll
        for (int cn = 0; cn < 16; cn++)
#pragma unroll
          for (int e = 0; e < 4; e++)
            o[cn][e] = __fmaf_rn(o[cn][e], sgn, __shfl_xor_sync(kFullMask, o[cn][e], 1 << st));
      }
    }
#pragma unroll
    for (int hh = 1; hh < 16; hh *= 2) {
      if (8 * hh < block) {
#pragma unroll
        for (int cn = 0; cn < 16; cn++)
          if (!(cn & hh))
#pragma unroll
            for (int e = 0; e < 4; e++) {
              const float a = o[cn][e], d = o[cn + hh][e];
              o[cn][e] = a + d;
              o[cn + hh][e] = a - d;
            }
      }
    }
  }
  const int ta = tok_first + r0 / G, tb = tok_first + r1 / G;
  __half* out0 = p.out + ((static_cast<size_t>(cq0) + ta) * p.num_kv_heads * G + h * G + r0 % G) * kD;
  __half* out1 = p.out + ((static_cast<size_t>(cq0) + tb) * p.num_kv_heads * G + h * G + r1 % G) * kD;
#pragma unroll
  for (int cn = 0; cn < 16; cn++) {
    if (ta < C)
      *reinterpret_cast<__half2*>(out0 + 8 * cn + 2 * c) =
          __floats2half2_rn(o[cn][0] * p.cb, o[cn][1] * p.cb);
    if (tb < C)
      *reinterpret_cast<__half2*>(out1 + 8 * cn + 2 * c) =
          __floats2half2_rn(o[cn][2] * p.cb, o[cn][3] * p.cb);
  }
  if (dead && w == 0) {
    // Let copies still in flight (issued by this warp, never waited for) land before the
    // CTA's shared memory is released; warp 0 stopped issuing when it gave up.
    for (int j = done0; j < issued; j++)
      mbar_wait_bounded(full_s + 8 * (j % kStagesP), static_cast<uint32_t>((j / kStagesP) & 1),
                        kWaitNs);
  }
}

template <int G, int SEFF>
void* prefill_ptr(bool fp4) {
  return fp4 ? reinterpret_cast<void*>(&prefill_kernel<G, SEFF, true>)
             : reinterpret_cast<void*>(&prefill_kernel<G, SEFF, false>);
}

void* pick_prefill(int group, int seff, bool fp4) {
#define KVQ_PICKP(GG)                                      \
  if (group == GG) {                                       \
    if (seff == 16) return prefill_ptr<GG, 16>(fp4);       \
    if (seff == 32) return prefill_ptr<GG, 32>(fp4);       \
  }
  KVQ_PICKP(1)
  KVQ_PICKP(2)
  KVQ_PICKP(4)
  KVQ_PICKP(8)
#undef KVQ_PICKP
  return nullptr;
}

size_t prefill_smem(int max_batch, bool fp4) {
  size_t s = static_cast<size_t>(kStagesP) * slot_bytes_p(fp4);  // ring
  s += fp4 ? 2 * 8 * kRows * 32 : 3 * 4 * kRows * 32;      // q: fp16 hi/lo or int8 slices
  s += sizeof(float) * kRows;                               // row scales
  s += (fp4 ? 4 : 2) * kTileTokens * 256;                   // fp16 V (and K) stages
  s += sizeof(uint64_t) * 2 * kStagesP;                     // barriers
  s += static_cast<size_t>(max_batch + 1) * sizeof(int32_t);  // query-block prefix
  s += 128;                                                  // alignment slack
  return (s + 15) & ~static_cast<size_t>(15);
}

}  // namespace

int launch_prefill(const PrefillParams& p, int total_q, cudaStream_t stream) {
  const int seff = p.page_size < kTileTokens ? p.page_size : kTileTokens;
  void* fn = pick_prefill(p.group, seff, p.fp4 != 0);
  if (!fn) return -1;
  if (p.batch == 0 || total_q == 0) return 0;
  const int QB = kRows / p.group;
  const long long blocks = (static_cast<long long>(total_q) + QB - 1) / QB + p.batch;
  const long long grid = blocks * p.num_kv_heads;
  if (grid > 0x7fffffffLL) return -1;
  const size_t smem = prefill_smem(p.batch, p.fp4 != 0);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(prefill_smem(4096, p.fp4 != 0))) != cudaSuccess)
    return -2;
  PrefillParams q = p;
  q.total_q = total_q;
  void* args[] = {&q};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreadsP);
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

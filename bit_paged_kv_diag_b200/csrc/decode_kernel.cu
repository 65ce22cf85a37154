// decode_kernel.cu -- paged GQA decode attention over the rotated INT4 cache, sm_100a.
//
// Method: "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化"
// (youngju.dev), section "KVキャッシュこそが本当のボトルネックである理由" (paged memory
// layout, regular access, fused attention execution) and section "回転のトリック —
// ブロック対角アダマール" (the rotation is orthogonal, so q.k is unchanged when both are
// rotated, and the rotation is undone exactly on the output).  Every decode step streams
// the whole cache, so the kernel is HBM-bound; everything below serves keeping the bytes
// moving with few instructions per byte.
//
// Work split (one launch).  The cache is cut into tiles of 32 tokens of one (sequence,
// KV head) "unit", numbered unit-major.  CTA k takes the contiguous tile range
// [k*chunk, (k+1)*chunk) of the T tiles, chunk = ceil(T/C), so every CTA streams the
// same number of bytes whatever the length mix.  Its 4 warps take the range's tiles in
// turn (tile X0 + w, X0 + w + 4, ...), each keeping an online-softmax state per unit; at
// the end of each unit the warps merge through shared memory.  A unit inside one CTA is finished
// there (normalise, inverse rotation, fp16 store).  A unit spanning several CTAs leaves
// one (o', m, l) partial per CTA in scratch slot unit + k (unique along the staircase of
// ranges); the last CTA to arrive (an atomic counter per unit, reset after use) merges
// them and finishes the unit.  The rotated, sliced q of a unit is prepared once per CTA
// (warp w takes query w) into a shared table the warps load their fragments from.
//
// Loads.  Each warp owns a ring of 3 shared-memory slots of one tile each.  Per tile one
// lane per page issues a 1-D bulk copy (cp.async.bulk, TMA engine, no multicast) of the
// contiguous (page, head) block -- codes and scales together -- into a slot, completing
// on the slot's mbarrier.  Page ids are read in batches, one per lane, a batch ahead of
// use, and sequence lengths are kept in shared memory, so no global-memory latency sits
// between consuming a tile and issuing the copy that refills its slot.
//
// QK^T on tensor cores in exact integer arithmetic: mma.sync m16n8k32 s8 x s8 -> s32 with
// A = K codes (16 tokens x 32 channels) and B = the rotated, scaled q cut into three int8
// slices, q' = M/64 * (q1 + q2/128 + q3/16384) with M the power of two above max|q'| (so
// q' is carried to 2^-21 of M).  A nibble becomes an int8 of value 16n with one or two
// bit operations (shift the nibble to the byte's top).  The channel order inside each
// k32 step is chosen so that a thread's fragment is one 32-bit word of codes (a dot
// product does not depend on the order of its terms).
// PV on tensor cores: mma.sync m16n8k16 f16 x f16 -> f32 with A = V codes transposed
// (16 channels x 16 tokens, gathered with byte permutes, exact fp16 integers) and B = P'
// = p * s_v (the V scale folded into the probabilities) as fp16 hi + lo parts: for G <= 4
// the two parts sit in neighbouring columns, for G = 8 two MMAs accumulate them.  (The
// integer values go in exactly, without a constant offset: the tensor core's internal
// sum is not precise enough to cancel a large offset afterwards.)  The GQA group is the N = 8
// side of both products; the dequantised cache is the M side.  The K scale multiplies the
// fp32 score of its token; softmax runs in the log2 domain with exp2.
//
// NVFP4 cache (template argument FP4; "BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号"
// (sns.style): E2M1 codes with an E4M3 scale per 16 channels, 144-byte token rows): the
// same work split, rings and merges; K and V are dequantised exactly to fp16 (hardware
// E2M1 / E4M3 conversions and one fp16 multiply), both products run as f16 mma.sync, and q
// is carried as fp16 hi + lo parts (tile_qk4, tile_pv4, prep_q4_warp).
#include <cuda_fp16.h>
#include <math_constants.h>
#include <stdint.h>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kD = 128;
// Token row of a (page, head) block: codes, then scales (INT4: one fp16 per K/V row;
// NVFP4: one E4M3 per 16 channels), and the ring slot of one tile.
constexpr int row_bytes(bool fp4) { return fp4 ? kD + kD / 8 : kD + 4; }
constexpr int slot_bytes(bool fp4) { return kTileTokens * row_bytes(fp4); }
constexpr int kWarps = kDecodeWarps;                // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 3;                          // ring slots per warp
constexpr uint64_t kWaitLimitNs = 2000000000ull;    // bounded waits: 2 s
constexpr unsigned kFull = 0xffffffffu;
constexpr float kMagic = 12582912.0f;               // 1.5 * 2^23

__device__ __forceinline__ int clamp_len(int L, int cap, int32_t* status) {
  if (L < 0 || L > cap) {
    atomicOr(status, KVQ_DEV_BAD_POS_BIT);
    return L < 0 ? 0 : cap;
  }
  return L;
}

// One (sequence, KV head) unit and its place in the tile sequence.  pre[] (tiles per
// sequence, exclusive prefix) and lens[] (clamped lengths) live in shared memory.
struct Unit {
  int b, h;  // sequence, KV head
  int n;     // tiles in the unit
  int L;     // tokens
  int U;     // global index of the unit's first tile
};

__device__ __forceinline__ void unit_of_tile(Unit& u, int x, const int32_t* pre, const int32_t* lens,
                                             const DecodeParams& p) {
  int lo = 0, hi = p.batch;  // pre[lo]*Hkv <= x < pre[hi]*Hkv
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pre[mid] * p.num_kv_heads <= x) lo = mid; else hi = mid;
  }
  u.b = lo;
  u.n = pre[lo + 1] - pre[lo];
  const int base = pre[lo] * p.num_kv_heads;
  u.h = (x - base) / u.n;
  u.U = base + u.h * u.n;
  u.L = lens[lo];
}

// The next non-empty unit.  Callers only ask while one exists.
__device__ __forceinline__ void unit_next(Unit& u, const int32_t* pre, const int32_t* lens,
                                          const DecodeParams& p) {
  if (++u.h == p.num_kv_heads) {
    u.h = 0;
    do { ++u.b; } while (u.b < p.batch && pre[u.b + 1] == pre[u.b]);
    if (u.b >= p.batch) return;
    u.n = pre[u.b + 1] - pre[u.b];
    u.L = lens[u.b];
  }
  u.U = pre[u.b] * p.num_kv_heads + u.h * u.n;
}

// ------------------------------------------------------------------- copies --
// Page entries of a warp's upcoming tiles, one per lane: a batch covers kBatch tiles of
// kPPT pages (tile t of the warp = CTA tile X0 + w + kWarps*t).  Entry lane: tile
// tb + lane / kPPT, page lane % kPPT of the tile, as the address of that (page, head)
// block with flags in its low 4 bits (blocks are 16-byte aligned): bits 0-2 = the
// tile's first token in the page / 32 (pages of 64+ tokens), bit 3 = the page id was out
// of range (page 0 is read instead and the status word is flagged at issue); 0 where no
// page is needed.
template <int SEFF>
struct PageBatch {
  static constexpr int kPPT = (SEFF < kTileTokens) ? kTileTokens / SEFF : 1;
  static constexpr int kBatch = 32 / kPPT;
};

constexpr uint64_t kEntryBad = 8u;

template <int SEFF, bool FP4>
__device__ __forceinline__ uint64_t load_page_batch(int tb, int X0, int X1, int w, int lane,
                                                    const int32_t* pre, const int32_t* lens,
                                                    const DecodeParams& p) {
  constexpr int kPPT = PageBatch<SEFF>::kPPT;
  const int x = X0 + w + kWarps * (tb + lane / kPPT);
  uint64_t e = 0;
  if (x < X1) {
    Unit u;
    unit_of_tile(u, x, pre, lens, p);
    const int t0 = (x - u.U) * kTileTokens;
    const int lp = (t0 >> p.page_shift) + lane % kPPT;
    if ((lp << p.page_shift) < u.L) {
      int pid = __ldg(p.page_table + static_cast<size_t>(u.b) * p.max_pages_per_seq + lp);
      uint64_t flags = 0;
      if (pid < 0 || pid >= p.num_pages) {
        pid = 0;
        flags = kEntryBad;
      }
      const size_t blk_bytes = static_cast<size_t>(p.page_size) * row_bytes(FP4);
      e = reinterpret_cast<uint64_t>(p.pool_layer +
                                     (static_cast<size_t>(pid) * p.num_kv_heads + u.h) * blk_bytes);
      if (SEFF == kTileTokens) e |= static_cast<uint64_t>((t0 & (p.page_size - 1)) / kTileTokens);
      e |= flags;
    }
  }
  return e;
}

// Issue the bulk copies of one tile into a ring slot (the whole warp calls; lane j <
// kPPT holds the tile's page entry j).  The slot holds a virtual page of SEFF = min(S, 32)
// token slots per copied page, [K codes][V codes][K scales][V scales], the pool's own
// block layout.
template <int SEFF, bool FP4>
__device__ __forceinline__ void tile_issue(uint64_t e, uint32_t slot, uint32_t bar, int lane,
                                           uint64_t pol, const DecodeParams& p) {
  constexpr int kPPT = PageBatch<SEFF>::kPPT;
  const bool have = lane < kPPT && e != 0;
  if (__any_sync(kFull, have && (e & kEntryBad)) && lane == 0) atomicOr(p.status, KVQ_DEV_BAD_PAGE_BIT);
  const int S = p.page_size;
  if (SEFF < kTileTokens || S == kTileTokens) {
    const uint8_t* blk = reinterpret_cast<const uint8_t*>(e & ~static_cast<uint64_t>(15));
    const uint32_t blk_bytes = static_cast<uint32_t>(S) * row_bytes(FP4);
    const int npg = __popc(__ballot_sync(kFull, have));
    if (lane == 0) mbar_arrive_expect_tx(bar, npg * blk_bytes);
    __syncwarp();
    if (have) bulk_copy_g2s(slot + lane * blk_bytes, blk, blk_bytes, bar, pol);
  } else {
    // One page per tile; lanes 0-3 copy its K codes, V codes, K scales and V scales.
    const uint64_t e0 = __shfl_sync(kFull, e, 0);
    const uint8_t* blk = reinterpret_cast<const uint8_t*>(e0 & ~static_cast<uint64_t>(15));
    const size_t o = static_cast<size_t>(e0 & 7u) * kTileTokens;  // tile's first token in the page
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
    if (lane == 0) mbar_arrive_expect_tx(bar, slot_bytes(FP4));
    __syncwarp();
    if (lane < 4) bulk_copy_g2s(dst, src, bytes, bar, pol);
  }
}

// A warp's producer: issues its tiles t = 0, 1, ... (CTA tile X0 + w + kWarps*t) in
// order into its ring, slot t % kStages; page entries come from batches loaded one
// batch ahead.
template <int SEFF, bool FP4>
struct Producer {
  int t;         // next tile to issue
  int nT;        // tiles of this warp
  int tb;        // first tile of the current batch
  uint64_t cur;  // this lane's entry of the current batch
  uint64_t nxt;  // ... of the next batch
};

template <int SEFF, bool FP4>
__device__ __forceinline__ void producer_issue(Producer<SEFF, FP4>& pr, int X0, int X1, int w, int lane,
                                               uint32_t ring_s, uint32_t bar_s, uint64_t pol,
                                               const int32_t* pre, const int32_t* lens,
                                               const DecodeParams& p) {
  constexpr int kPPT = PageBatch<SEFF>::kPPT, kBatch = PageBatch<SEFF>::kBatch;
  if (pr.t >= pr.tb + kBatch) {
    pr.tb += kBatch;
    pr.cur = pr.nxt;
    pr.nxt = pr.tb + kBatch < pr.nT ? load_page_batch<SEFF, FP4>(pr.tb + kBatch, X0, X1, w, lane, pre, lens, p) : 0;
  }
  const int src = (pr.t - pr.tb) * kPPT + lane;
  const uint64_t e = __shfl_sync(kFull, pr.cur, src & 31);
  const int s = pr.t % kStages;
  tile_issue<SEFF, FP4>(e, ring_s + s * slot_bytes(FP4), bar_s + 8 * s, lane, pol, p);
  pr.t++;
}

// ------------------------------------------------------------------------ q --
// int8 B fragments of the rotated, scaled q, per k32 chunk jj: [jj][0] = k 4c..4c+3,
// [jj][1] = k 16+4c..16+4c+3, where k = 4c + e <-> channel 32c + 8jj + 2e and
// k = 16 + 4c + e <-> channel 32c + 8jj + 2e + 1.
// G <= 4: A = column g holds slice 1 (g even) or 2 (g odd) of query g/2, B = slice 3
// (g even) or zero.  G == 8: A, B, C = slices 1, 2, 3 of query g.
template <int G>
struct QFrag {
  static constexpr int NQ = (G == 8) ? 2 : 1;  // queries owned by one thread
  uint32_t A[4][2], B[4][2], C[4][2];
  float sf[NQ];  // M / 1024 of the owned queries
};

// Rotate (the fixed-order butterfly: stages h = 1, 2 in registers, h = 4..64 across
// lanes), scale by c_b * softmax_scale * log2(e), and cut every query of the unit into
// three int8 slices q' = M/64 * (q1 + q2/128 + q3/16384), M the power of two >= max|q'|
// (1 for a zero row).  qraw: the unit's G fp16 rows in shared memory; the slices go to the
// warp's fragment table in fragment order:
//   frag word ((qi*3 + s)*4 + c)*8 + 2*jj + half, byte e  <->  channel 32c + 8jj + 2e + half.
// The warp prepares queries q0, q0 + QSTEP, ... < G (all of them for QSTEP = 1; a
// quarter each when the CTA's warps share one unit's rows).
// Rotated, scaled queries qb, qb + QSTEP, ... (QB of them; indices past G repeat the last
// one and are not stored by the callers): x[b][e] = channel 4*lane + e, and the power of
// two M[b] >= max |q'| (1 for a zero row).
template <int G, int QSTEP, int QB>
__device__ __forceinline__ void rotate_q(const uint8_t* qraw, int qb, int lane, const DecodeParams& p,
                                       float (&x)[QB][4], float (&M)[QB]) {
#pragma unroll
  for (int b = 0; b < QB; b++) {
    const int qi = min(qb + b * QSTEP, G - 1);  // a clamped duplicate is computed, not stored
    const uint2 raw = *reinterpret_cast<const uint2*>(qraw + qi * kD * 2 + 8 * lane);
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    const float t0 = lo.x, t1 = lo.y, t2 = hi.x, t3 = hi.y;
    const float a0 = __fadd_rn(t0, t1), a1 = __fsub_rn(t0, t1);
    const float a2 = __fadd_rn(t2, t3), a3 = __fsub_rn(t2, t3);
    const bool rot = p.hadamard_block > 1;  // b = 1 (plain INT4): no rotation
    x[b][0] = rot ? __fadd_rn(a0, a2) : t0;
    x[b][2] = rot ? __fsub_rn(a0, a2) : t2;
    x[b][1] = rot ? __fadd_rn(a1, a3) : t1;
    x[b][3] = rot ? __fsub_rn(a1, a3) : t3;
  }
#pragma unroll
  for (int s = 0; s < 5; s++) {
    if ((4 << s) < p.hadamard_block) {
      const float sgn = ((lane >> s) & 1) ? -1.0f : 1.0f;
#pragma unroll
      for (int b = 0; b < QB; b++)
#pragma unroll
        for (int e = 0; e < 4; e++)
          x[b][e] = __fmaf_rn(x[b][e], sgn, __shfl_xor_sync(kFull, x[b][e], 1 << s));
    }
  }
  float amax[QB];
#pragma unroll
  for (int b = 0; b < QB; b++) {
    amax[b] = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; e++) {
      x[b][e] = __fmul_rn(__fmul_rn(x[b][e], p.cb), p.q_scale);
      amax[b] = fmaxf(amax[b], fabsf(x[b][e]));
    }
  }
#pragma unroll
  for (int d = 1; d < 32; d *= 2)
#pragma unroll
    for (int b = 0; b < QB; b++) amax[b] = fmaxf(amax[b], __shfl_xor_sync(kFull, amax[b], d));
#pragma unroll
  for (int b = 0; b < QB; b++) {
    M[b] = 1.0f;
    if (amax[b] > 1e-30f) {
      const uint32_t bits = __float_as_uint(amax[b]);
      M[b] = (bits & 0x7FFFFFu) ? __uint_as_float((bits & 0x7F800000u) + 0x00800000u) : amax[b];
    }
  }
}

template <int G, int QSTEP>
__device__ __forceinline__ void prep_q_warp(const uint8_t* qraw, uint32_t* frag, float* sf, int lane,
                                            const DecodeParams& p, int q0 = 0) {
  // Up to four queries at a time: their shuffle chains are independent and interleave.
  constexpr int NQW = (G + QSTEP - 1) / QSTEP;
  constexpr int QB = NQW < 4 ? NQW : 4;
  const int c = lane >> 3, jj = (lane >> 1) & 3, e0 = (2 * lane) & 3;
  uint8_t* base = reinterpret_cast<uint8_t*>(frag);
#pragma unroll 1
  for (int qb = q0; qb < G; qb += QB * QSTEP) {
    float x[QB][4];
#pragma unroll
    for (int b = 0; b < QB; b++) {
      const int qi = min(qb + b * QSTEP, G - 1);  // a clamped duplicate is computed, not stored
      const uint2 raw = *reinterpret_cast<const uint2*>(qraw + qi * kD * 2 + 8 * lane);
      const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
      const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
      const float t0 = lo.x, t1 = lo.y, t2 = hi.x, t3 = hi.y;
      const float a0 = __fadd_rn(t0, t1), a1 = __fsub_rn(t0, t1);
      const float a2 = __fadd_rn(t2, t3), a3 = __fsub_rn(t2, t3);
      const bool rot = p.hadamard_block > 1;  // b = 1 (plain INT4): no rotation
      x[b][0] = rot ? __fadd_rn(a0, a2) : t0;
      x[b][2] = rot ? __fsub_rn(a0, a2) : t2;
      x[b][1] = rot ? __fadd_rn(a1, a3) : t1;
      x[b][3] = rot ? __fsub_rn(a1, a3) : t3;
    }
#pragma unroll
    for (int s = 0; s < 5; s++) {
      if ((4 << s) < p.hadamard_block) {
        const float sgn = ((lane >> s) & 1) ? -1.0f : 1.0f;
#pragma unroll
        for (int b = 0; b < QB; b++)
#pragma unroll
          for (int e = 0; e < 4; e++)
            x[b][e] = __fmaf_rn(x[b][e], sgn, __shfl_xor_sync(kFull, x[b][e], 1 << s));
      }
    }
    float amax[QB];
#pragma unroll
    for (int b = 0; b < QB; b++) {
      amax[b] = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; e++) {
        x[b][e] = __fmul_rn(__fmul_rn(x[b][e], p.cb), p.q_scale);
        amax[b] = fmaxf(amax[b], fabsf(x[b][e]));
      }
    }
#pragma unroll
    for (int d = 1; d < 32; d *= 2)
#pragma unroll
      for (int b = 0; b < QB; b++) amax[b] = fmaxf(amax[b], __shfl_xor_sync(kFull, amax[b], d));
#pragma unroll
    for (int b = 0; b < QB; b++) {
      float M = 1.0f;
      if (amax[b] > 1e-30f) {
        const uint32_t bits = __float_as_uint(amax[b]);
        M = (bits & 0x7FFFFFu) ? __uint_as_float((bits & 0x7F800000u) + 0x00800000u) : amax[b];
      }
      const float inv = __fdiv_rn(64.0f, M);  // exact: powers of two
      uint32_t ms[3][4];
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const float t = x[b][e] * inv;                      // |t| <= 64, exact scaling
        const float m1 = t + kMagic;                        // rint(t) in the low mantissa bits
        const float r1 = (t - (m1 - kMagic)) * 128.0f;      // exact
        const float m2 = r1 + kMagic;
        const float r2 = (r1 - (m2 - kMagic)) * 128.0f;
        const float m3 = r2 + kMagic;
        ms[0][e] = __float_as_uint(m1);
        ms[1][e] = __float_as_uint(m2);
        ms[2][e] = __float_as_uint(m3);
      }
      // Channels 4*lane + i: c = lane/8, jj = (lane/2)%4, half = i%2, byte e0 + i/2 with
      // e0 = (2*lane)%4: a 2-byte store per (slice, half).
      const int qi = qb + b * QSTEP;
      if (qi >= G) continue;
#pragma unroll
      for (int sl = 0; sl < 3; sl++) {
        const int word = ((qi * 3 + sl) * 4 + c) * 8 + 2 * jj;
        const uint16_t h0 = static_cast<uint16_t>((ms[sl][0] & 0xFFu) | ((ms[sl][2] & 0xFFu) << 8));
        const uint16_t h1 = static_cast<uint16_t>((ms[sl][1] & 0xFFu) | ((ms[sl][3] & 0xFFu) << 8));
        *reinterpret_cast<uint16_t*>(base + word * 4 + e0) = h0;
        *reinterpret_cast<uint16_t*>(base + (word + 1) * 4 + e0) = h1;
      }
      if (lane == 0) sf[qi] = M * (1.0f / 1024.0f);
    }
  }
  __syncwarp();
}

template <int G>
__device__ __forceinline__ void qfrag_load(QFrag<G>& f, const uint32_t* qfb, const float* sfb,
                                           int lane) {
  const int g = lane >> 2, c = lane & 3;
  const int qi = (G == 8) ? g : (g >> 1);
  const bool ok = qi < G;
  uint4 s[3][2];
#pragma unroll
  for (int sl = 0; sl < 3; sl++) {
    s[sl][0] = s[sl][1] = make_uint4(0u, 0u, 0u, 0u);
    if (ok) {
      const uint4* src = reinterpret_cast<const uint4*>(qfb + ((qi * 3 + sl) * 4 + c) * 8);
      s[sl][0] = src[0];
      s[sl][1] = src[1];
    }
  }
#pragma unroll
  for (int jj = 0; jj < 4; jj++)
#pragma unroll
    for (int e = 0; e < 2; e++) {
      uint32_t v[3];
#pragma unroll
      for (int sl = 0; sl < 3; sl++) {
        const uint4 q4 = s[sl][jj >> 1];
        const uint32_t wds[4] = {q4.x, q4.y, q4.z, q4.w};
        v[sl] = wds[2 * (jj & 1) + e];
      }
      if (G == 8) {
        f.A[jj][e] = v[0];
        f.B[jj][e] = v[1];
        f.C[jj][e] = v[2];
      } else {
        f.A[jj][e] = (g & 1) ? v[1] : v[0];
        f.B[jj][e] = (g & 1) ? 0u : v[2];
        f.C[jj][e] = 0u;
      }
    }
  if (G == 8) {
    f.sf[0] = sfb[2 * c];
    f.sf[QFrag<G>::NQ - 1] = sfb[2 * c + 1];
  } else {
    f.sf[0] = c < G ? sfb[c] : 1.0f;
  }
}

// ---------------------------------------------------------------- NVFP4 q --
// NVFP4 cache ("BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号" (sns.style): E2M1 codes
// with an E4M3 scale per 16 channels).  K and V are dequantised to fp16 exactly (an E2M1
// value times an E4M3 scale has at most 6 significant bits and lies in [2^-10, 2688]);
// QK^T and PV run as mma.sync m16n8k16 f16 x f16 -> f32.  q' is normalised by M (the
// power of two >= max |q'|) to |q~| <= 2^14 and carried as fp16 hi + lo parts (about
// 2^-22 relative).  Fragment table row (qi, part) = 128 fp16 in channel order.
template <int G, int QSTEP>
__device__ __forceinline__ void prep_q4_warp(const uint8_t* qraw, uint32_t* frag, float* sf, int lane,
                                             const DecodeParams& p, int q0 = 0) {
  constexpr int NQW = (G + QSTEP - 1) / QSTEP;
  constexpr int QB = NQW < 4 ? NQW : 4;
  __half* base = reinterpret_cast<__half*>(frag);
#pragma unroll 1
  for (int qb = q0; qb < G; qb += QB * QSTEP) {
    float x[QB][4], Mq[QB];
    rotate_q<G, QSTEP, QB>(qraw, qb, lane, p, x, Mq);
#pragma unroll
    for (int b = 0; b < QB; b++) {
      const int qi = qb + b * QSTEP;
      if (qi >= G) continue;
      const float inv = __fdiv_rn(16384.0f, Mq[b]);  // exact: powers of two
      __half hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const float t = x[b][e] * inv;
        hi[e] = __float2half_rn(t);
        lo[e] = __float2half_rn(t - __half2float(hi[e]));
      }
      *reinterpret_cast<uint2*>(base + (qi * 2) * kD + 4 * lane) =
          make_uint2(pack_half2(hi[0], hi[1]), pack_half2(hi[2], hi[3]));
      *reinterpret_cast<uint2*>(base + (qi * 2 + 1) * kD + 4 * lane) =
          make_uint2(pack_half2(lo[0], lo[1]), pack_half2(lo[2], lo[3]));
      if (lane == 0) sf[qi] = Mq[b] * (1.0f / 16384.0f);
    }
  }
  __syncwarp();
}

// f16 B fragments of q~ per k-step kk (16 channels: k rows 2c + e <-> channel
// 32c + 4kk + e, k rows 2c + 8 + e <-> channel 32c + 4kk + 2 + e), column g.
// G <= 4: column g holds part g & 1 (hi, lo) of query g / 2 in H; G == 8: H and L are the
// hi and lo parts of query g.
template <int G>
struct QFrag4 {
  static constexpr int NQ = (G == 8) ? 2 : 1;
  uint32_t H[8][2];
  uint32_t L[G == 8 ? 8 : 1][2];
  float sf[NQ];
};

template <int G>
__device__ __forceinline__ void qfrag4_load(QFrag4<G>& f, const uint32_t* qfb, const float* sfb,
                                            int lane) {
  const int g = lane >> 2, c = lane & 3;
  const int qi = (G == 8) ? g : (g >> 1);
  const bool ok = qi < G;
  const int row_h = (G == 8) ? 2 * g : 2 * qi + (g & 1);
#pragma unroll
  for (int part = 0; part < (G == 8 ? 2 : 1); part++) {
    uint4 w[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
      w[i] = make_uint4(0u, 0u, 0u, 0u);
      if (ok) w[i] = reinterpret_cast<const uint4*>(qfb + (row_h + part) * (kD / 2) + 16 * c)[i];
    }
#pragma unroll
    for (int kk = 0; kk < 8; kk++) {
      const uint4 q4 = w[kk >> 1];
      const uint32_t a = (kk & 1) ? q4.z : q4.x, b = (kk & 1) ? q4.w : q4.y;
      if (part == 0) {
        f.H[kk][0] = a;
        f.H[kk][1] = b;
      } else {
        f.L[G == 8 ? kk : 0][0] = a;
        f.L[G == 8 ? kk : 0][1] = b;
      }
    }
  }
  if (G == 8) {
    f.sf[0] = sfb[2 * c];
    f.sf[QFrag4<G>::NQ - 1] = sfb[2 * c + 1];
  } else {
    f.sf[0] = c < G ? sfb[c] : 1.0f;
  }
}

// The 4 bytes of w, each two E2M1 codes (low nibble first) -> 4 x fp16x2, exact.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&d)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(w));
}

// Two E4M3 scale bytes (low 16 bits, low byte first) -> fp16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t b) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(b)));
  return h;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Scores (log2 domain) of an NVFP4 tile, in tile_qk's layout: A row g <-> token tau0,
// row g + 8 <-> tau1; the lane's 16 code bytes of a token row are channels 32c..32c+31
// (blocks 2c, 2c + 1), byte 2kk <-> channels 32c + 4kk, +1 (k columns 2c, 2c + 1).
template <int G, int SEFF>
__device__ __forceinline__ void tile_qk4(const QFrag4<G>& qf, const uint8_t* slot, int ntok, int lane,
                                         float (&sc)[2][QFrag4<G>::NQ][2]) {
  constexpr int RB = row_bytes(true);
  const int g = lane >> 2, c = lane & 3;
  const int tau0 = (g < 4) ? g : g + 4;
  const int tau1 = tau0 + 4;
#pragma unroll
  for (int j = 0; j < 2; j++) {
    const uint8_t* pbase = slot + (16 * j / SEFF) * (SEFF * RB);
    const int sl = (16 * j) % SEFF;
    const uint4 ka = *reinterpret_cast<const uint4*>(pbase + (sl + tau0) * 64 + 16 * c);
    const uint4 kc = *reinterpret_cast<const uint4*>(pbase + (sl + tau1) * 64 + 16 * c);
    const uint32_t sa = *reinterpret_cast<const uint16_t*>(pbase + SEFF * 128 + (sl + tau0) * 8 + 2 * c);
    const uint32_t sc2 = *reinterpret_cast<const uint16_t*>(pbase + SEFF * 128 + (sl + tau1) * 8 + 2 * c);
    const uint32_t fa = e4m3x2_to_f16x2(sa), fc = e4m3x2_to_f16x2(sc2);
    const uint32_t sA[2] = {prmt(fa, fa, 0x1010u), prmt(fa, fa, 0x3232u)};
    const uint32_t sC[2] = {prmt(fc, fc, 0x1010u), prmt(fc, fc, 0x3232u)};
    const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w};
    const uint32_t wc[4] = {kc.x, kc.y, kc.z, kc.w};
    float accH[4] = {0.0f, 0.0f, 0.0f, 0.0f}, accL[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int wi = 0; wi < 4; wi++) {  // word wi = k-steps 2wi, 2wi + 1
      uint32_t da[4], dc[4];
      e2m1x8_to_f16x2(wa[wi], da);
      e2m1x8_to_f16x2(wc[wi], dc);
      const int blk = wi >> 1;  // k-steps 0-3: block 2c; 4-7: block 2c + 1
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int kk = 2 * wi + h;
        const uint32_t a0 = hmul2(da[2 * h], sA[blk]), a2 = hmul2(da[2 * h + 1], sA[blk]);
        const uint32_t a1 = hmul2(dc[2 * h], sC[blk]), a3 = hmul2(dc[2 * h + 1], sC[blk]);
        mma_16816(accH, a0, a1, a2, a3, qf.H[kk][0], qf.H[kk][1]);
        if (G == 8) mma_16816(accL, a0, a1, a2, a3, qf.L[G == 8 ? kk : 0][0], qf.L[G == 8 ? kk : 0][1]);
      }
    }
    const bool v0 = 16 * j + tau0 < ntok, v1 = 16 * j + tau1 < ntok;
    if (G == 8) {
#pragma unroll
      for (int qq = 0; qq < 2; qq++)
#pragma unroll
        for (int r = 0; r < 2; r++) {
          const int e = 2 * r + qq;
          sc[j][qq][r] = (r ? v1 : v0) ? (accH[e] + accL[e]) * qf.sf[qq] : -CUDART_INF_F;
        }
    } else {
      // Column 2c = hi part, 2c + 1 = lo part of query c.
      sc[j][0][0] = v0 ? (accH[0] + accH[1]) * qf.sf[0] : -CUDART_INF_F;
      sc[j][0][1] = v1 ? (accH[2] + accH[3]) * qf.sf[0] : -CUDART_INF_F;
    }
  }
}

// ------------------------------------------------------------------- state --
template <int G>
struct State {
  static constexpr int NQ = QFrag<G>::NQ;
  float o[8][4];  // PV accumulators: m-tile i = channels 16g+2i (rows g) and 16g+2i+1
  float m[NQ];
  float l[NQ];
};

template <int G>
__device__ __forceinline__ void state_reset(State<G>& st) {
#pragma unroll
  for (int i = 0; i < 8; i++)
#pragma unroll
    for (int e = 0; e < 4; e++) st.o[i][e] = 0.0f;
#pragma unroll
  for (int qq = 0; qq < State<G>::NQ; qq++) {
    st.m[qq] = -CUDART_INF_F;
    st.l[qq] = 0.0f;
  }
}


// One tile = 2 k-steps of 16 tokens in a ring slot (a shared-memory pointer); ntok
// valid tokens.  The work is split in three so that the QK^T of the next tile and the
// PV of the current one sit in one straight-line block the compiler can interleave.

// Scores (log2 domain) of the tile: sc[k-step][owned query][row], -inf past ntok.
template <int G, int SEFF>
__device__ __forceinline__ void tile_qk(const QFrag<G>& qf, const uint8_t* slot, int ntok, int lane,
                                        float (&sc)[2][QFrag<G>::NQ][2]) {
  const int g = lane >> 2, c = lane & 3;
  const int tau0 = (g < 4) ? g : g + 4;  // token of A row g
  const int tau1 = tau0 + 4;             // token of A row g + 8
#pragma unroll
  for (int j = 0; j < 2; j++) {
    const uint8_t* pbase = slot + (16 * j / SEFF) * (SEFF * 132);
    const int sl = (16 * j) % SEFF;
    const uint4 ka = *reinterpret_cast<const uint4*>(pbase + (sl + tau0) * 64 + 16 * c);
    const uint4 kc = *reinterpret_cast<const uint4*>(pbase + (sl + tau1) * 64 + 16 * c);
    const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w};
    const uint32_t wc[4] = {kc.x, kc.y, kc.z, kc.w};
    int accA[4] = {0, 0, 0, 0}, accB[4] = {0, 0, 0, 0}, accC[4] = {0, 0, 0, 0};
#pragma unroll
    for (int jj = 0; jj < 4; jj++) {
      const uint32_t a0 = (wa[jj] << 4) & 0xF0F0F0F0u, a1 = (wc[jj] << 4) & 0xF0F0F0F0u;
      const uint32_t a2 = wa[jj] & 0xF0F0F0F0u, a3 = wc[jj] & 0xF0F0F0F0u;
      mma_16832_s8(accA, a0, a1, a2, a3, qf.A[jj][0], qf.A[jj][1]);
      mma_16832_s8(accB, a0, a1, a2, a3, qf.B[jj][0], qf.B[jj][1]);
      if (G == 8) mma_16832_s8(accC, a0, a1, a2, a3, qf.C[jj][0], qf.C[jj][1]);
    }
    const __half* skp = reinterpret_cast<const __half*>(pbase + SEFF * 128) + sl;
    const float sk0 = __half2float(skp[tau0]), sk1 = __half2float(skp[tau1]);
    const bool v0 = 16 * j + tau0 < ntok, v1 = 16 * j + tau1 < ntok;
    const float k14 = 1.0f / 16384.0f;
    if (G == 8) {
      // Column 2c = query 2c (qq 0), 2c+1 = query 2c+1 (qq 1); rows g (d0, d1), g+8 (d2, d3).
#pragma unroll
      for (int qq = 0; qq < 2; qq++)
#pragma unroll
        for (int r = 0; r < 2; r++) {
          const int e = 2 * r + qq;
          const float v = static_cast<float>(accA[e]) + static_cast<float>(accB[e] * 128 + accC[e]) * k14;
          sc[j][qq][r] = (r ? v1 : v0) ? v * ((r ? sk1 : sk0) * qf.sf[qq]) : -CUDART_INF_F;
        }
    } else {
      // Column 2c = slices 1 (A) and 3 (B) of query c, 2c+1 = slice 2 (A) of query c.
      const float va = static_cast<float>(accA[0]) + static_cast<float>(accA[1] * 128 + accB[0]) * k14;
      const float vc = static_cast<float>(accA[2]) + static_cast<float>(accA[3] * 128 + accB[2]) * k14;
      sc[j][0][0] = v0 ? va * (sk0 * qf.sf[0]) : -CUDART_INF_F;
      sc[j][0][1] = v1 ? vc * (sk1 * qf.sf[0]) : -CUDART_INF_F;
    }
  }
}

// Online softmax update with the tile's scores, in two parts.  The statistics part moves
// m and l to the tile's frame and turns sc into p = exp2(score - m); it leaves the o'
// accumulators alone, so it can run next to the previous tile's PV.  The rescale part
// then brings o' to the new frame (alpha = exp2(m_old - m_new)).
template <int G>
__device__ __forceinline__ bool tile_softmax_stats(State<G>& st, float (&sc)[2][QFrag<G>::NQ][2],
                                                   float (&alpha)[QFrag<G>::NQ]) {
  constexpr int NQ = State<G>::NQ;
  bool rescale = false;
#pragma unroll
  for (int qq = 0; qq < NQ; qq++) {
    float mx = fmaxf(fmaxf(sc[0][qq][0], sc[0][qq][1]), fmaxf(sc[1][qq][0], sc[1][qq][1]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
    const float mnew = fmaxf(st.m[qq], mx);
    alpha[qq] = ex2_approx(st.m[qq] - mnew);
    rescale |= alpha[qq] != 1.0f;
    st.m[qq] = mnew;
    float ps = 0.0f;
#pragma unroll
    for (int j = 0; j < 2; j++)
#pragma unroll
      for (int r = 0; r < 2; r++) {
        sc[j][qq][r] = ex2_approx(sc[j][qq][r] - mnew);
        ps += sc[j][qq][r];
      }
    st.l[qq] = st.l[qq] * alpha[qq] + ps;
  }
  return __any_sync(kFull, rescale);
}

template <int G>
__device__ __forceinline__ void tile_rescale(State<G>& st, const float (&alpha)[QFrag<G>::NQ]) {
  constexpr int NQ = State<G>::NQ;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    // G <= 4: columns 2c, 2c+1 are query c's hi and lo parts; G == 8: queries 2c, 2c+1.
    st.o[i][0] *= alpha[0];
    st.o[i][2] *= alpha[0];
    st.o[i][1] *= alpha[NQ - 1];
    st.o[i][3] *= alpha[NQ - 1];
  }
}

// (p0, p1) -> fp16 pairs hi = rn(p), lo = rn(p - hi): p carried to about 2^-22.
__device__ __forceinline__ void split_hi_lo(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(p0, p1);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(p0 - f.x, p1 - f.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// PV of the tile with probabilities pr.  B fragment of thread (g, c): tokens c, c+4 (b0)
// and c+8, c+12 (b1) of the k-step for column g, taken from the lanes that scored them
// (rows c and c + 4 of the QK^T fragment).
template <int G, int SEFF>
__device__ __forceinline__ void tile_pv(State<G>& st, const uint8_t* slot, int ntok, int lane,
                                        const float (&pr)[2][QFrag<G>::NQ][2]) {
  const int g = lane >> 2, c = lane & 3;
  const int tau0 = (g < 4) ? g : g + 4;
  const int tau1 = tau0 + 4;
  const int srcA = 4 * c + (g >> 1);
  const int srcB = srcA + 16;
#pragma unroll
  for (int j = 0; j < 2; j++) {
    const uint8_t* pbase = slot + (16 * j / SEFF) * (SEFF * 132);
    const int sl = (16 * j) % SEFF;
    const uint8_t* vb = pbase + SEFF * 64 + sl * 64;
    const __half* svp = reinterpret_cast<const __half*>(pbase + SEFF * 130) + sl;
    const float sv0 = __half2float(svp[tau0]), sv1 = __half2float(svp[tau1]);
    const bool v0 = 16 * j + tau0 < ntok, v1 = 16 * j + tau1 < ntok;
    // P' = p * s_v carried as fp16 hi + lo (relative precision ~2^-22).
    uint32_t bh0, bh1, bl0 = 0u, bl1 = 0u;
    if (G == 8) {
      uint32_t xh[2], xl[2];
#pragma unroll
      for (int qq = 0; qq < 2; qq++) {
        const float p0 = v0 ? pr[j][qq][0] * sv0 : 0.0f, p1 = v1 ? pr[j][qq][1] * sv1 : 0.0f;
        split_hi_lo(p0, p1, xh[qq], xl[qq]);
      }
      // Column g = query g, owned by lane group c' = g/2 as its query (g & 1).
      const uint32_t aE = __shfl_sync(kFull, xh[0], srcA), aO = __shfl_sync(kFull, xh[1], srcA);
      const uint32_t cE = __shfl_sync(kFull, xh[0], srcB), cO = __shfl_sync(kFull, xh[1], srcB);
      const uint32_t dE = __shfl_sync(kFull, xl[0], srcA), dO = __shfl_sync(kFull, xl[1], srcA);
      const uint32_t eE = __shfl_sync(kFull, xl[0], srcB), eO = __shfl_sync(kFull, xl[1], srcB);
      bh0 = (g & 1) ? aO : aE;
      bh1 = (g & 1) ? cO : cE;
      bl0 = (g & 1) ? dO : dE;
      bl1 = (g & 1) ? eO : eE;
    } else {
      const float p0 = v0 ? pr[j][0][0] * sv0 : 0.0f, p1 = v1 ? pr[j][0][1] * sv1 : 0.0f;
      uint32_t xh, xl;
      split_hi_lo(p0, p1, xh, xl);
      // Column g = 2q + part holds query q's hi (part 0) or lo (part 1) part.
      const uint32_t aH = __shfl_sync(kFull, xh, srcA), aL = __shfl_sync(kFull, xl, srcA);
      const uint32_t cH = __shfl_sync(kFull, xh, srcB), cL = __shfl_sync(kFull, xl, srcB);
      bh0 = (g & 1) ? aL : aH;
      bh1 = (g & 1) ? cL : cH;
      if ((g >> 1) >= G) bh0 = bh1 = 0u;
    }
    // V rows of tokens c, c+4, c+8, c+12; this thread's channels [16g, 16g+16).
    const uint2 t0 = *reinterpret_cast<const uint2*>(vb + (c + 0) * 64 + 8 * g);
    const uint2 t1 = *reinterpret_cast<const uint2*>(vb + (c + 4) * 64 + 8 * g);
    const uint2 t2 = *reinterpret_cast<const uint2*>(vb + (c + 8) * 64 + 8 * g);
    const uint2 t3 = *reinterpret_cast<const uint2*>(vb + (c + 12) * 64 + 8 * g);
    const uint32_t w0[2] = {t0.x, t0.y}, w1[2] = {t1.x, t1.y};
    const uint32_t w2[2] = {t2.x, t2.y}, w3[2] = {t3.x, t3.y};
#pragma unroll
    for (int i = 0; i < 8; i++) {  // m-tile i: byte i of the chunk = channels 16g+2i, +1
      const uint32_t e = i & 3;
      const uint32_t sel = e | (e << 4) | ((4 + e) << 8) | ((4 + e) << 12);
      const uint32_t r01 = prmt(w0[i >> 2], w1[i >> 2], sel);
      const uint32_t r23 = prmt(w2[i >> 2], w3[i >> 2], sel);
      const uint32_t a0 = nib_lo_to_half2(r01), a1 = nib_hi_to_half2(r01);
      const uint32_t a2 = nib_lo_to_half2(r23), a3 = nib_hi_to_half2(r23);
      mma_16816(st.o[i], a0, a1, a2, a3, bh0, bh1);
      if (G == 8) mma_16816(st.o[i], a0, a1, a2, a3, bl0, bl1);
    }
  }
}

// Bytes 0 and 2 of w, each two E2M1 codes (low nibble first) -> 2 x fp16x2, exact.
__device__ __forceinline__ void e2m1x2_b02_to_f16x2(uint32_t w, uint32_t& d0, uint32_t& d2) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b2;\n\t}"
      : "=r"(d0), "=r"(d2)
      : "r"(w));
}

// (a & m) | (b & ~m)
__device__ __forceinline__ uint32_t bitsel(uint32_t a, uint32_t b, uint32_t m) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(r) : "r"(a), "r"(b), "r"(m));
  return r;
}

// PV of an NVFP4 tile with probabilities pr: as tile_pv, with P' = p; the V scales are
// applied in the dequantised A operand (the lane's channels 16g..16g+15 are block g of
// each token row, so a register's two tokens each take their own scale).
template <int G, int SEFF>
__device__ __forceinline__ void tile_pv4(State<G>& st, const uint8_t* slot, int ntok, int lane,
                                         const float (&pr)[2][QFrag4<G>::NQ][2]) {
  constexpr int RB = row_bytes(true);
  const int g = lane >> 2, c = lane & 3;
  const int tau0 = (g < 4) ? g : g + 4;
  const int tau1 = tau0 + 4;
  const int srcA = 4 * c + (g >> 1);
  const int srcB = srcA + 16;
#pragma unroll
  for (int j = 0; j < 2; j++) {
    const uint8_t* pbase = slot + (16 * j / SEFF) * (SEFF * RB);
    const int sl = (16 * j) % SEFF;
    const uint8_t* vb = pbase + SEFF * 64 + sl * 64;
    const uint8_t* vs = pbase + SEFF * 128 + SEFF * 8 + sl * 8;  // V scales [token][8]
    const bool v0 = 16 * j + tau0 < ntok, v1 = 16 * j + tau1 < ntok;
    uint32_t bh0, bh1, bl0 = 0u, bl1 = 0u;
    if (G == 8) {
      uint32_t xh[2], xl[2];
#pragma unroll
      for (int qq = 0; qq < 2; qq++) {
        const float p0 = v0 ? pr[j][qq][0] : 0.0f, p1 = v1 ? pr[j][qq][1] : 0.0f;
        split_hi_lo(p0, p1, xh[qq], xl[qq]);
      }
      const uint32_t aE = __shfl_sync(kFull, xh[0], srcA), aO = __shfl_sync(kFull, xh[1], srcA);
      const uint32_t cE = __shfl_sync(kFull, xh[0], srcB), cO = __shfl_sync(kFull, xh[1], srcB);
      const uint32_t dE = __shfl_sync(kFull, xl[0], srcA), dO = __shfl_sync(kFull, xl[1], srcA);
      const uint32_t eE = __shfl_sync(kFull, xl[0], srcB), eO = __shfl_sync(kFull, xl[1], srcB);
      bh0 = (g & 1) ? aO : aE;
      bh1 = (g & 1) ? cO : cE;
      bl0 = (g & 1) ? dO : dE;
      bl1 = (g & 1) ? eO : eE;
    } else {
      const float p0 = v0 ? pr[j][0][0] : 0.0f, p1 = v1 ? pr[j][0][1] : 0.0f;
      uint32_t xh, xl;
      split_hi_lo(p0, p1, xh, xl);
      const uint32_t aH = __shfl_sync(kFull, xh, srcA), aL = __shfl_sync(kFull, xl, srcA);
      const uint32_t cH = __shfl_sync(kFull, xh, srcB), cL = __shfl_sync(kFull, xl, srcB);
      bh0 = (g & 1) ? aL : aH;
      bh1 = (g & 1) ? cL : cH;
      if ((g >> 1) >= G) bh0 = bh1 = 0u;
    }
    // V rows of tokens c, c+4, c+8, c+12; this thread's channels [16g, 16g+16) = block g.
    const uint2 t0 = *reinterpret_cast<const uint2*>(vb + (c + 0) * 64 + 8 * g);
    const uint2 t1 = *reinterpret_cast<const uint2*>(vb + (c + 4) * 64 + 8 * g);
    const uint2 t2 = *reinterpret_cast<const uint2*>(vb + (c + 8) * 64 + 8 * g);
    const uint2 t3 = *reinterpret_cast<const uint2*>(vb + (c + 12) * 64 + 8 * g);
    // Tokens past the sequence's end take scale 0: their slot bytes are whatever the pool or
    // an earlier tile left there, and an E4M3 NaN would survive the zero probability.
    const int t0n = 16 * j + c;
    const uint32_t s0 = t0n < ntok ? vs[(c + 0) * 8 + g] : 0u, s1 = t0n + 4 < ntok ? vs[(c + 4) * 8 + g] : 0u;
    const uint32_t s2 = t0n + 8 < ntok ? vs[(c + 8) * 8 + g] : 0u, s3 = t0n + 12 < ntok ? vs[(c + 12) * 8 + g] : 0u;
    const uint32_t s01 = s0 | (s1 << 8), s23 = s2 | (s3 << 8);
    const uint32_t S01 = e4m3x2_to_f16x2(s01), S23 = e4m3x2_to_f16x2(s23);
    const uint32_t w0[2] = {t0.x, t0.y}, w1[2] = {t1.x, t1.y};
    const uint32_t w2[2] = {t2.x, t2.y}, w3[2] = {t3.x, t3.y};
#pragma unroll
    for (int i = 0; i < 8; i += 2) {  // m-tiles i, i + 1: bytes e, e + 1 of word i / 4
      const uint32_t e = i & 3;
      // bytes: [row0 byte e, row1 byte e, row0 byte e+1, row1 byte e+1]
      const uint32_t sel = e | ((4 + e) << 4) | ((e + 1) << 8) | ((5 + e) << 12);
      const uint32_t X01 = prmt(w0[i >> 2], w1[i >> 2], sel);
      const uint32_t X23 = prmt(w2[i >> 2], w3[i >> 2], sel);
      // even channels: low nibbles of the two tokens; odd: high nibbles (bytes 0 and 2)
      const uint32_t ev01 = bitsel(X01, X01 >> 4, 0x000F000Fu), od01 = bitsel(X01 >> 4, X01 >> 8, 0x000F000Fu);
      const uint32_t ev23 = bitsel(X23, X23 >> 4, 0x000F000Fu), od23 = bitsel(X23 >> 4, X23 >> 8, 0x000F000Fu);
      uint32_t a0[2], a1[2], a2[2], a3[2];
      e2m1x2_b02_to_f16x2(ev01, a0[0], a0[1]);
      e2m1x2_b02_to_f16x2(od01, a1[0], a1[1]);
      e2m1x2_b02_to_f16x2(ev23, a2[0], a2[1]);
      e2m1x2_b02_to_f16x2(od23, a3[0], a3[1]);
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const uint32_t A0 = hmul2(a0[h], S01), A1 = hmul2(a1[h], S01);
        const uint32_t A2 = hmul2(a2[h], S23), A3 = hmul2(a3[h], S23);
        mma_16816(st.o[i + h], A0, A1, A2, A3, bh0, bh1);
        if (G == 8) mma_16816(st.o[i + h], A0, A1, A2, A3, bl0, bl1);
      }
    }
  }
}

// Warp partial of one unit (its owned queries) -> a record block [G][kPartStride] at rec
// (shared or global memory): o'[128], m, l per query.  With qsel >= 0 only query qsel is
// written, at rec itself.
template <int G>
__device__ __forceinline__ void state_write(const State<G>& st, float* rec, int lane, int qsel = -1) {
  constexpr int NQ = State<G>::NQ;
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int qq = 0; qq < NQ; qq++) {
    float l = st.l[qq];
    l += __shfl_xor_sync(kFull, l, 4);
    l += __shfl_xor_sync(kFull, l, 8);
    l += __shfl_xor_sync(kFull, l, 16);
    const int qi = (G == 8) ? 2 * c + qq : c;
    if (qi >= G || (qsel >= 0 && qi != qsel)) continue;
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; i++) {
      if (G == 8) {
        v[2 * i] = st.o[i][qq];
        v[2 * i + 1] = st.o[i][2 + qq];
      } else {  // hi + lo columns
        v[2 * i] = st.o[i][0] + st.o[i][1];
        v[2 * i + 1] = st.o[i][2] + st.o[i][3];
      }
    }
    float* r = rec + (qsel >= 0 ? 0 : qi * kPartStride);
    float4* dst = reinterpret_cast<float4*>(r + 16 * g);
#pragma unroll
    for (int e = 0; e < 4; e++) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    if (g == 0) {
      r[kD] = st.m[qq];
      r[kD + 1] = l;
    }
  }
}

// o'/l of one query (lane: channels 4*lane..4*lane+3) -> inverse block-diagonal
// Hadamard -> fp16 store.
__device__ __forceinline__ void finish_query(const float (&o)[4], float l, __half* dst, int lane,
                                             const DecodeParams& p) {
  float x[4];
  const float rl = __frcp_rn(l);
#pragma unroll
  for (int e = 0; e < 4; e++) x[e] = o[e] * rl;
  const int block = p.hadamard_block;
  {
    const bool rot = block > 1;  // b = 1 (plain INT4): no rotation
    const float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
    x[0] = rot ? a0 + a2 : x[0];
    x[1] = rot ? a1 + a3 : x[1];
    x[2] = rot ? a0 - a2 : x[2];
    x[3] = rot ? a1 - a3 : x[3];
  }
#pragma unroll
  for (int s = 0; s < 5; s++) {
    if ((4 << s) < block) {
      const int bit = 1 << s;
      const float sgn = (lane & bit) ? -1.0f : 1.0f;
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const float other = __shfl_xor_sync(kFull, x[e], bit);
        x[e] = __fmaf_rn(x[e], sgn, other);
      }
    }
  }
  const uint32_t lo = pack_half2(__float2half_rn(x[0] * p.cb), __float2half_rn(x[1] * p.cb));
  const uint32_t hi = pack_half2(__float2half_rn(x[2] * p.cb), __float2half_rn(x[3] * p.cb));
  *reinterpret_cast<uint2*>(dst + 4 * lane) = make_uint2(lo, hi);
}

// A unit with a single contributing warp (one tile): finish it from the warp's registers,
// one query at a time through a staging area of kPartStride floats.
template <int G>
__device__ __forceinline__ void finish_from_state(const State<G>& st, float* stage, __half* orow,
                                                  int lane, const DecodeParams& p) {
#pragma unroll 1
  for (int qi = 0; qi < G; qi++) {
    __syncwarp();
    state_write<G>(st, stage, lane, qi);
    __syncwarp();
    const float4 v = *reinterpret_cast<const float4*>(stage + 4 * lane);
    const float o[4] = {v.x, v.y, v.z, v.w};
    finish_query(o, stage[kD + 1], orow + qi * kD, lane, p);
  }
  __syncwarp();
}

template <bool GLOBAL>
__device__ __forceinline__ float2 ld_rec2(const float* a) {
  if (GLOBAL) return __ldcg(reinterpret_cast<const float2*>(a));
  return *reinterpret_cast<const float2*>(a);
}
template <bool GLOBAL>
__device__ __forceinline__ float4 ld_rec4(const float* a) {
  if (GLOBAL) return __ldcg(reinterpret_cast<const float4*>(a));
  return *reinterpret_cast<const float4*>(a);
}

// Merge of at most RMAX records (the common case: a unit's CTAs or a CTA's warps): every
// lane loads the (m, l) pairs and its o' slice of all records for two of the warp's queries
// at once (the (m, l) loads are broadcasts), so two queries cost one round trip and no
// cross-lane reduction.  Same contract as merge_records below.
template <int G, int QSTEP, bool GLOBAL, int RMAX, typename F>
__device__ __forceinline__ void merge_few(int nrec, F&& rec, int q0, __half* orow, float* crec,
                                          int lane, const DecodeParams& p) {
  constexpr int NQW = (G + QSTEP - 1) / QSTEP;  // queries this warp handles (at most)
  constexpr int QB = NQW < 2 ? NQW : 2;          // queries per round trip
#pragma unroll 1
  for (int qb = q0; qb < G; qb += QB * QSTEP) {
    float2 ml[QB][RMAX];
    float4 v[QB][RMAX];
#pragma unroll
    for (int i = 0; i < QB; i++) {
      const int qi = qb + i * QSTEP;
#pragma unroll
      for (int r = 0; r < RMAX; r++) {
        ml[i][r] = make_float2(-CUDART_INF_F, 0.0f);
        v[i][r] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (r < nrec && qi < G) {
          const float* rr = rec(r) + qi * kPartStride;
          ml[i][r] = ld_rec2<GLOBAL>(rr + kD);
          v[i][r] = ld_rec4<GLOBAL>(rr + 4 * lane);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < QB; i++) {
      const int qi = qb + i * QSTEP;
      if (qi >= G) continue;
      float M = ml[i][0].x;
#pragma unroll
      for (int r = 1; r < RMAX; r++) M = fmaxf(M, ml[i][r].x);
      float o[4] = {0.0f, 0.0f, 0.0f, 0.0f}, l = 0.0f;
#pragma unroll
      for (int r = 0; r < RMAX; r++) {
        const float e = (ml[i][r].x == -CUDART_INF_F) ? 0.0f : ex2_approx(ml[i][r].x - M);
        l += e * ml[i][r].y;
        o[0] += e * v[i][r].x;
        o[1] += e * v[i][r].y;
        o[2] += e * v[i][r].z;
        o[3] += e * v[i][r].w;
      }
      if (crec) {
        float* r = crec + qi * kPartStride;
        *reinterpret_cast<float4*>(r + 4 * lane) = make_float4(o[0], o[1], o[2], o[3]);
        if (lane == 0) *reinterpret_cast<float2*>(r + kD) = make_float2(M, l);
      } else {
        finish_query(o, l, orow + qi * kD, lane, p);
      }
    }
  }
}

// Merge nrec partial records of one unit (record j: [G][kPartStride] floats at rec(j)) for
// the queries q0, q0 + QSTEP, ... < G (one warp; lane: channels 4*lane..4*lane+3), then
// either finish them into orow or, with crec != nullptr, store the merged record there.
// Records are taken 32 at a time with an online rescale: lane j fetches (m, l) of record j
// of the chunk for every owned query, in the same round as the o' rows of the chunk's
// first records (8 float4 per lane a round), so a merge of a few records costs one round
// trip to L2.
// GLOBAL: the records were written by other warps or CTAs and are read from L2.
template <int G, int QSTEP, bool GLOBAL, typename F>
__device__ __forceinline__ void merge_records(int nrec, F&& rec, int q0, __half* orow, float* crec,
                                              int lane, const DecodeParams& p) {
  constexpr int NQW = (G + QSTEP - 1) / QSTEP;       // queries this warp handles (at most)
  constexpr int R = (8 / NQW) < 1 ? 1 : 8 / NQW;     // records per round of o' loads
  if (q0 >= G) return;
  float M[NQW], l[NQW], o[NQW][4];
#pragma unroll
  for (int i = 0; i < NQW; i++) {
    M[i] = -CUDART_INF_F;
    l[i] = 0.0f;
    o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  }
  for (int base = 0; base < nrec; base += 32) {
    const bool mine = base + lane < nrec;
    const float* rj = mine ? rec(base + lane) : nullptr;
    const int cnt = min(32, nrec - base);
    // o' rows of records base .. base + R - 1, fetched together with the (m, l) pairs.
    float4 v[R][NQW];
    auto fetch = [&](int j0) {
#pragma unroll
      for (int r = 0; r < R; r++) {
        const int j = j0 + r;
        const float* rr = (j < cnt) ? rec(base + j) : nullptr;
#pragma unroll
        for (int i = 0; i < NQW; i++) {
          const int qi = min(q0 + i * QSTEP, G - 1);
          v[r][i] = rr ? ld_rec4<GLOBAL>(rr + qi * kPartStride + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    };
    fetch(0);
    float e[NQW];
    float2 ml[NQW];
#pragma unroll
    for (int i = 0; i < NQW; i++) {
      const int qi = min(q0 + i * QSTEP, G - 1);
      ml[i] = mine ? ld_rec2<GLOBAL>(rj + qi * kPartStride + kD) : make_float2(-CUDART_INF_F, 0.0f);
    }
#pragma unroll
    for (int i = 0; i < NQW; i++) {
      float mc = ml[i].x;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) mc = fmaxf(mc, __shfl_xor_sync(kFull, mc, d));
      const float Mn = fmaxf(M[i], mc);  // finite: every record holds at least one token
      const float r = (M[i] == -CUDART_INF_F) ? 0.0f : exp2f(M[i] - Mn);
      M[i] = Mn;
      l[i] *= r;
#pragma unroll
      for (int c = 0; c < 4; c++) o[i][c] *= r;
      e[i] = (ml[i].x == -CUDART_INF_F) ? 0.0f : exp2f(ml[i].x - Mn);
      float le = e[i] * ml[i].y;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) le += __shfl_xor_sync(kFull, le, d);
      l[i] += le;
    }
    for (int j0 = 0; j0 < cnt; j0 += R) {
      if (j0 > 0) fetch(j0);
#pragma unroll
      for (int r = 0; r < R; r++) {
#pragma unroll
        for (int i = 0; i < NQW; i++) {
          const float ej = __shfl_sync(kFull, e[i], (j0 + r) & 31);  // 0 past cnt: v is 0 too
          o[i][0] += ej * v[r][i].x;
          o[i][1] += ej * v[r][i].y;
          o[i][2] += ej * v[r][i].z;
          o[i][3] += ej * v[r][i].w;
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < NQW; i++) {
    const int qi = q0 + i * QSTEP;
    if (qi >= G) continue;
    if (crec) {
      float* r = crec + qi * kPartStride;
      *reinterpret_cast<float4*>(r + 4 * lane) = make_float4(o[i][0], o[i][1], o[i][2], o[i][3]);
      if (lane == 0) *reinterpret_cast<float2*>(r + kD) = make_float2(M[i], l[i]);
    } else {
      finish_query(o[i], l[i], orow + qi * kD, lane, p);
    }
  }
}

// --------------------------------------------------------- fused append --
// One new token of one (sequence, KV head): its K or V row rotated and quantised by a
// warp, bit-identical to the append kernel (the fixed-order butterfly: stages h = 1, 2
// inside a lane's 4 channels, h = 4..64 across lanes as fma(own, +-1, other), one rounding
// each; then y = fl(y * c_b); s = fp16(fl(max|y| / 7)); codes = round-half-even of y / s
// decided exactly by comparing y with (k + 1/2) * s, clamped to [-8, 7]).  Lane L gets the
// 16 code bits of channels 4L..4L+3 (low nibble = even channel) and the fp16 scale bits.
struct NewRow {
  uint32_t codes16;  // this lane's 2 bytes of the packed row
  uint32_t scale;    // fp16 bits, same in every lane
};

__device__ __forceinline__ uint2 load_new_row(const __half* row, int lane) {
  return __ldg(reinterpret_cast<const uint2*>(row) + lane);  // channels 4*lane..4*lane+3
}

// The rotated row y = fl(c_b * butterfly(x)) of channels 4*lane..4*lane+3.
__device__ __forceinline__ void rotate_new_row(uint2 raw, int lane, const DecodeParams& p, float (&x)[4]) {
  const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
  const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
  x[0] = lo.x;
  x[1] = lo.y;
  x[2] = hi.x;
  x[3] = hi.y;
  if (p.hadamard_block > 1) {
    const float a0 = __fadd_rn(x[0], x[1]), a1 = __fsub_rn(x[0], x[1]);
    const float a2 = __fadd_rn(x[2], x[3]), a3 = __fsub_rn(x[2], x[3]);
    x[0] = __fadd_rn(a0, a2);
    x[2] = __fsub_rn(a0, a2);
    x[1] = __fadd_rn(a1, a3);
    x[3] = __fsub_rn(a1, a3);
#pragma unroll
    for (int st = 0; st < 5; st++) {
      if ((4 << st) < p.hadamard_block) {
        const float sgn = ((lane >> st) & 1) ? -1.0f : 1.0f;
#pragma unroll
        for (int e = 0; e < 4; e++) x[e] = __fmaf_rn(x[e], sgn, __shfl_xor_sync(kFull, x[e], 1 << st));
      }
    }
#pragma unroll
    for (int e = 0; e < 4; e++) x[e] = __fmul_rn(x[e], p.cb);
  }
}

__device__ __forceinline__ NewRow quantise_new_row(uint2 raw, int lane, const DecodeParams& p) {
  float x[4];
  rotate_new_row(raw, lane, p, x);
  float m = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int d = 1; d < 32; d *= 2) m = fmaxf(m, __shfl_xor_sync(kFull, m, d));
  const float s32 = __fdiv_rn(m, 7.0f);
  const __half sh = s32 > 65504.0f ? __ushort_as_half(0x7BFF) : __float2half_rn(s32);
  const float s = __half2float(sh);
  NewRow r;
  r.scale = __half_as_ushort(sh);
  r.codes16 = 0u;
  if (s != 0.0f) {
    const float rc = __frcp_rn(s), hs = 0.5f * s;
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const float k = floorf(__fmul_rn(x[e], rc));
      const float h = __fmaf_rn(k, s, hs);  // (k + 1/2) * s, exact
      const bool odd = (__float_as_uint(__fadd_rn(k, kMagic)) & 1u) != 0u;
      const bool up = x[e] > h || (x[e] == h && odd);
      const int c = static_cast<int>(fminf(fmaxf(up ? k + 1.0f : k, -8.0f), 7.0f));
      r.codes16 |= (static_cast<uint32_t>(c) & 0xFu) << (4 * e);
    }
  }
  return r;
}

// NVFP4 new row, bit-identical to the append kernel: lanes 4m..4m+3 hold block m (16
// channels); s = E4M3(fl(max |y| / 6)) (nearest even, saturating), codes = E2M1(fl(y *
// fl(1/s))) (nearest even, saturating, sign kept), 0 when s == 0.  codes16 = the lane's two
// code bytes; scale = block m's E4M3 byte (the same in its 4 lanes).
__device__ __forceinline__ NewRow quantise_new_row_fp4(uint2 raw, int lane, const DecodeParams& p) {
  float x[4];
  rotate_new_row(raw, lane, p, x);
  float m = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
  m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
  uint16_t sb2;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(sb2) : "f"(0.0f), "f"(__fdiv_rn(m, 6.0f)));
  const uint32_t sh = e4m3x2_to_f16x2(sb2);
  const float s = __half2float(__ushort_as_half(static_cast<uint16_t>(sh & 0xFFFFu)));
  NewRow r;
  r.scale = sb2 & 0xFFu;
  r.codes16 = 0u;
  if (s != 0.0f) {
    const float rc = __frcp_rn(s);
    uint32_t b0, b1;
    asm("{\n\t.reg .b8 q;\n\tcvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\tcvt.u32.u8 %0, q;\n\t}"
        : "=r"(b0) : "f"(__fmul_rn(x[1], rc)), "f"(__fmul_rn(x[0], rc)));
    asm("{\n\t.reg .b8 q;\n\tcvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\tcvt.u32.u8 %0, q;\n\t}"
        : "=r"(b1) : "f"(__fmul_rn(x[3], rc)), "f"(__fmul_rn(x[2], rc)));
    r.codes16 = b0 | (b1 << 8);
  }
  return r;
}

// Bytes of a token's scales in a block row (K, then V) and the patch buffer's layout:
// [K codes 64 B][V codes 64 B][K scales][V scales], then the token's place in its tile.
template <bool FP4>
struct PatchLayout {
  static constexpr int kScale = FP4 ? kD / 16 : 2;   // per K or V row
  static constexpr int kJ = 128 + 2 * kScale;          // 132 or 144
};

// The new token of a unit (its raw K and V rows kraw, vraw as loaded by load_new_row):
// rotate and quantise the rows into the warp's patch buffer (shared memory), in the block
// layout of one token.
template <bool FP4>
__device__ __forceinline__ void fused_quantise(uint2 kraw, uint2 vraw, int lane, uint8_t* patch,
                                               const DecodeParams& p) {
  if constexpr (FP4) {
    const NewRow kr = quantise_new_row_fp4(kraw, lane, p);
    const NewRow vr = quantise_new_row_fp4(vraw, lane, p);
    *reinterpret_cast<uint16_t*>(patch + 2 * lane) = static_cast<uint16_t>(kr.codes16);
    *reinterpret_cast<uint16_t*>(patch + 64 + 2 * lane) = static_cast<uint16_t>(vr.codes16);
    if ((lane & 3) == 0) {
      patch[128 + (lane >> 2)] = static_cast<uint8_t>(kr.scale);
      patch[136 + (lane >> 2)] = static_cast<uint8_t>(vr.scale);
    }
  } else {
    const NewRow kr = quantise_new_row(kraw, lane, p);
    const NewRow vr = quantise_new_row(vraw, lane, p);
    *reinterpret_cast<uint16_t*>(patch + 2 * lane) = static_cast<uint16_t>(kr.codes16);
    *reinterpret_cast<uint16_t*>(patch + 64 + 2 * lane) = static_cast<uint16_t>(vr.codes16);
    if (lane == 0) {
      *reinterpret_cast<uint16_t*>(patch + 128) = static_cast<uint16_t>(kr.scale);
      *reinterpret_cast<uint16_t*>(patch + 130) = static_cast<uint16_t>(vr.scale);
    }
  }
  __syncwarp();
}

// Store the patch buffer's token of unit (b, h) at position seq_lens[b] of the pool
// (skipped, with the status flagged, when the position or its page is out of range).
// Returns whether it is stored and belongs in the decode.
template <bool FP4>
__device__ __forceinline__ bool fused_store(int b, int h, int lane, const uint8_t* patch,
                                            const DecodeParams& p) {
  constexpr int SC = PatchLayout<FP4>::kScale;
  const int pos = __ldg(p.seq_lens + b);
  const int S = p.page_size;
  const int lp = pos >> p.page_shift;
  if (pos < 0 || lp >= p.max_pages_per_seq) return false;  // flagged by the length clamp
  const int page = __ldg(p.page_table + static_cast<size_t>(b) * p.max_pages_per_seq + lp);
  if (page < 0 || page >= p.num_pages) return false;     // flagged when the tile is issued
  const int slot = pos & (S - 1);
  uint8_t* blk = const_cast<uint8_t*>(p.pool_layer) + (static_cast<size_t>(page) * p.num_kv_heads + h) *
                                      (static_cast<size_t>(S) * (kD + 2 * SC));
  const uint16_t kc = *reinterpret_cast<const uint16_t*>(patch + 2 * lane);
  const uint16_t vc = *reinterpret_cast<const uint16_t*>(patch + 64 + 2 * lane);
  *reinterpret_cast<uint16_t*>(blk + slot * 64 + 2 * lane) = kc;
  *reinterpret_cast<uint16_t*>(blk + S * 64 + slot * 64 + 2 * lane) = vc;
  if (lane == 0) {
    if constexpr (FP4) {
      *reinterpret_cast<uint2*>(blk + S * 128 + slot * 8) = *reinterpret_cast<const uint2*>(patch + 128);
      *reinterpret_cast<uint2*>(blk + S * 136 + slot * 8) = *reinterpret_cast<const uint2*>(patch + 136);
    } else {
      *reinterpret_cast<uint16_t*>(blk + S * 128 + slot * 2) = *reinterpret_cast<const uint16_t*>(patch + 128);
      *reinterpret_cast<uint16_t*>(blk + S * 130 + slot * 2) = *reinterpret_cast<const uint16_t*>(patch + 130);
    }
  }
  return true;
}

// Overwrite token j (0..31, kept at byte PatchLayout::kJ of the patch buffer) of a landed
// ring slot with the patch buffer's token (the slot's copy of the pool may predate the
// store above).  The warp syncs before the slot is read.
template <int SEFF, bool FP4>
__device__ __forceinline__ void patch_slot(uint8_t* slot, int lane, const uint8_t* patch) {
  constexpr int SC = PatchLayout<FP4>::kScale;
  const int j = *reinterpret_cast<const int*>(patch + PatchLayout<FP4>::kJ);  // place in the tile
  uint8_t* base = slot + (j / SEFF) * (SEFF * row_bytes(FP4));
  const int jj = j % SEFF;
  const uint32_t wv = reinterpret_cast<const uint32_t*>(patch)[lane];  // bytes 4*lane..
  uint8_t* dst = lane < 16 ? base + jj * 64 + 4 * lane : base + SEFF * 64 + jj * 64 + 4 * (lane - 16);
  *reinterpret_cast<uint32_t*>(dst) = wv;
  if (lane == 0) {
    if constexpr (FP4) {
      *reinterpret_cast<uint2*>(base + SEFF * 128 + jj * SC) = *reinterpret_cast<const uint2*>(patch + 128);
      *reinterpret_cast<uint2*>(base + SEFF * (128 + SC) + jj * SC) = *reinterpret_cast<const uint2*>(patch + 136);
    } else {
      *reinterpret_cast<uint16_t*>(base + SEFF * 128 + jj * 2) = *reinterpret_cast<const uint16_t*>(patch + 128);
      *reinterpret_cast<uint16_t*>(base + SEFF * 130 + jj * 2) = *reinterpret_cast<const uint16_t*>(patch + 130);
    }
  }
  __syncwarp();
}

// Per-warp fragment table: G queries x 96 words, at least one staging record.
// (NVFP4: G queries x 2 fp16 parts x 128 channels = G x 128 words.)
constexpr int frag_words(int g, bool fp4) {
  return (fp4 ? g * 128 : g * 96) > kPartStride ? (fp4 ? g * 128 : g * 96) : kPartStride;
}

// The format's q preparation, fragments and tile steps.
template <int G, int QSTEP, bool FP4>
__device__ __forceinline__ void prep_q(const uint8_t* qraw, uint32_t* frag, float* sf, int lane,
                                       const DecodeParams& p, int q0 = 0) {
  if constexpr (FP4) prep_q4_warp<G, QSTEP>(qraw, frag, sf, lane, p, q0);
  else prep_q_warp<G, QSTEP>(qraw, frag, sf, lane, p, q0);
}

template <int G, bool FP4>
struct QF {
  using type = QFrag<G>;
};
template <int G>
struct QF<G, true> {
  using type = QFrag4<G>;
};

template <int G>
__device__ __forceinline__ void qfrag_get(QFrag<G>& f, const uint32_t* qfb, const float* sfb, int lane) {
  qfrag_load<G>(f, qfb, sfb, lane);
}
template <int G>
__device__ __forceinline__ void qfrag_get(QFrag4<G>& f, const uint32_t* qfb, const float* sfb, int lane) {
  qfrag4_load<G>(f, qfb, sfb, lane);
}

template <int G, int SEFF>
__device__ __forceinline__ void tile_qk_any(const QFrag<G>& qf, const uint8_t* slot, int ntok, int lane,
                                            float (&sc)[2][QFrag<G>::NQ][2]) {
  tile_qk<G, SEFF>(qf, slot, ntok, lane, sc);
}
template <int G, int SEFF>
__device__ __forceinline__ void tile_qk_any(const QFrag4<G>& qf, const uint8_t* slot, int ntok, int lane,
                                            float (&sc)[2][QFrag4<G>::NQ][2]) {
  tile_qk4<G, SEFF>(qf, slot, ntok, lane, sc);
}

template <int G, int SEFF, bool FP4>
__device__ __forceinline__ void tile_pv_any(State<G>& st, const uint8_t* slot, int ntok, int lane,
                                            const float (&pr)[2][QFrag<G>::NQ][2]) {
  if constexpr (FP4) tile_pv4<G, SEFF>(st, slot, ntok, lane, pr);
  else tile_pv<G, SEFF>(st, slot, ntok, lane, pr);
}

// FUSED: the one-token append runs inside (p.k_new, p.v_new set).
// FP4: the cache holds NVFP4 rows.
template <int G, int SEFF, bool FUSED, bool FP4>
__global__ void __launch_bounds__(kThreads, 3) decode_kernel(DecodeParams p) {
  constexpr int kFragWords = frag_words(G, FP4);
  constexpr int kSlot = slot_bytes(FP4);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  // Bulk copies need 16-byte aligned destinations; align to 128 bytes (the allocation
  // carries 128 spare bytes for this).
  uint8_t* smem = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  uint8_t* ring = smem;                                                      // [w][stage][4224]
  // Per warp (index w) and two more for the CTA's first and last unit (indices kWarps,
  // kWarps + 1): raw q rows, fragment table, M factors.
  constexpr int kQT = kWarps + 2;
  uint8_t* qraw_all = ring + kWarps * kStages * kSlot;                       // [kQT][G][128] fp16
  uint32_t* frag_all = reinterpret_cast<uint32_t*>(qraw_all + kQT * G * kD * 2);  // [kQT][kFragWords]
  float* sf_all = reinterpret_cast<float*>(frag_all + kQT * kFragWords);     // [kQT][8]
  float* mbuf = sf_all + kQT * 8;                                            // [w][G][132]
  uint64_t* bars = reinterpret_cast<uint64_t*>(mbuf + kWarps * G * kPartStride);  // [w][kStages+1], CTA q
  int32_t* pre = reinterpret_cast<int32_t*>(bars + kWarps * (kStages + 1) + 1);  // [batch + 1]
  int32_t* lens = pre + p.batch + 1;                                         // [batch]
  __shared__ int warp_sum[kWarps];
  __shared__ int running;
  __shared__ int last_flag_e[2];

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int cap = p.max_pages_per_seq * p.page_size;
  // The prologue below reads only seq_lens and the page table, which no kernel of this
  // library writes (and may OR bits into the status word); everything else an earlier
  // kernel may write or read (pool, q, new K/V rows, out, the scratch) is touched only
  // after griddep_wait().
  griddep_launch_dependents();

  const uint32_t qbar_cta = smem_addr(bars + kWarps * (kStages + 1));
  if (tid == 0) {
    mbar_init(qbar_cta, 1);
    fence_mbar_init();
  }

  // Clamped lengths, and tiles per sequence -> exclusive prefix pre[0..batch].
  if (tid == 0) running = 0;
  __syncthreads();
  for (int base = 0; base < p.batch; base += kThreads) {
    const int i = base + tid;
    int n = 0;
    if (i < p.batch) {
      const int L = clamp_len(__ldg(p.seq_lens + i) + (FUSED ? 1 : 0), cap, p.status);
      lens[i] = L;
      n = (L + kTileTokens - 1) / kTileTokens;
    }
    int incl = n;
#pragma unroll
    for (int d = 1; d < 32; d *= 2) {
      const int y = __shfl_up_sync(kFull, incl, d);
      if (lane >= d) incl += y;
    }
    if (lane == 31) warp_sum[w] = incl;
    __syncthreads();
    int before = running;
    for (int w2 = 0; w2 < w; w2++) before += warp_sum[w2];
    if (i < p.batch) pre[i] = before + incl - n;
    __syncthreads();
    if (tid == kThreads - 1) running = before + incl;
    __syncthreads();
  }
  if (tid == 0) pre[p.batch] = running;
  __syncthreads();

  // CTA k takes tiles [k*chunk, (k+1)*chunk) of the T tiles (the host bounds T < 2^30);
  // warp w of it takes tiles X0 + w, X0 + w + kWarps, ...
  const int T = pre[p.batch] * p.num_kv_heads;
  const int chunk = (T + p.total_ctas - 1) / p.total_ctas;
  const int kc = blockIdx.x;
  const int X0 = kc * chunk;
  const int X1 = min(T, X0 + chunk);
  const bool has_tiles = T > 0 && X0 < T;

  uint8_t* qraw = qraw_all + w * G * kD * 2;
  uint32_t* frag = frag_all + w * kFragWords;
  float* sf = sf_all + w * 8;
  uint8_t* ring_w = ring + w * kStages * kSlot;
  const uint8_t* ring_p = ring_w;
  const uint32_t ring_s = smem_addr(ring_p);
  const uint32_t bar_s = smem_addr(bars + w * (kStages + 1));
  const uint32_t qbar = bar_s + 8 * kStages;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s <= kStages; s++) mbar_init(bar_s + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_policy_evict_first();

  // Producer: page-id batches 0 and 1 (page table only: before the wait).
  constexpr int kBatch = PageBatch<SEFF>::kBatch;
  Producer<SEFF, FP4> pr;
  pr.t = 0;
  pr.nT = has_tiles ? max(0, (X1 - X0 - w + kWarps - 1) / kWarps) : 0;
  pr.tb = 0;
  pr.cur = has_tiles ? load_page_batch<SEFF, FP4>(0, X0, X1, w, lane, pre, lens, p) : 0;
  pr.nxt = pr.nT > kBatch ? load_page_batch<SEFF, FP4>(kBatch, X0, X1, w, lane, pre, lens, p) : 0;

  // This warp's q rows of a unit: one bulk copy into its raw-q buffer, completing on qbar.
  int q_issued = 0, q_done = 0;  // q copies issued / waited for (one in flight at most)
  auto q_fetch = [&](const Unit& u) {
    q_issued++;
    if (lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(qbar, G * kD * 2);
      bulk_copy_g2s(smem_addr(qraw),
                    p.q + (static_cast<size_t>(u.b) * p.num_kv_heads * G + u.h * G) * kD,
                    G * kD * 2, qbar, 0ull);
    }
    __syncwarp();
  };
  // The units of the CTA's range: the first (uf) and the last (ul) may be shared with
  // other CTAs; the units between them lie wholly inside the range.
  Unit uf, ul;
  if (has_tiles) {
    unit_of_tile(uf, X0, pre, lens, p);
    unit_of_tile(ul, X1 - 1, pre, lens, p);
  }
  int x = X0 + w;
  Unit cu;
  if (x < X1) unit_of_tile(cu, x, pre, lens, p);
  // uf and ul have one copy of their q rows each, prepared by all warps together; only
  // units between them are prepared by the warp that walks them.
  auto is_uf = [&](const Unit& u) { return u.b == uf.b && u.h == uf.h; };
  auto is_ul = [&](const Unit& u) { return u.b == ul.b && u.h == ul.h; };
  const bool two_edges = has_tiles && !is_uf(ul);

  // Fused append: if this warp holds the last tile of its first unit and that unit's q
  // comes from a CTA table (its own fragment table is then free as the patch buffer), the
  // unit's new K/V rows are loaded, rotated and quantised before the wait -- the inputs
  // of an append are complete when the previous kernel lets this one start, and this is
  // pure arithmetic into shared memory; the pool store waits.  Other units do it at their
  // segment's start.
  bool pre_quantised = false;
  if constexpr (FUSED) {
    if (x < X1 && (is_uf(cu) || is_ul(cu))) {
      const int seg_end0 = min(X1, cu.U + cu.n);
      const int xl0 = x + kWarps * ((seg_end0 - x + kWarps - 1) / kWarps - 1);
      if (xl0 == cu.U + cu.n - 1) {
        const size_t row = (static_cast<size_t>(cu.b) * p.num_kv_heads + cu.h) * kD;
        fused_quantise<FP4>(load_new_row(p.k_new + row, lane), load_new_row(p.v_new + row, lane), lane,
                            reinterpret_cast<uint8_t*>(frag), p);
        pre_quantised = true;
      }
    }
  }

  griddep_wait();

  // q goes ahead of the tile copies, so that it is not queued behind them; then the first
  // kStages tiles.
  if (has_tiles && tid == 0) {
    mbar_arrive_expect_tx(qbar_cta, (two_edges ? 2 : 1) * G * kD * 2);
    bulk_copy_g2s(smem_addr(qraw_all + kWarps * G * kD * 2),
                  p.q + (static_cast<size_t>(uf.b) * p.num_kv_heads * G + uf.h * G) * kD,
                  G * kD * 2, qbar_cta, 0ull);
    if (two_edges)
      bulk_copy_g2s(smem_addr(qraw_all + (kWarps + 1) * G * kD * 2),
                    p.q + (static_cast<size_t>(ul.b) * p.num_kv_heads * G + ul.h * G) * kD,
                    G * kD * 2, qbar_cta, 0ull);
  }
  if (x < X1 && !is_uf(cu) && !is_ul(cu)) q_fetch(cu);
  while (pr.t < pr.nT && pr.t < kStages)
    producer_issue<SEFF, FP4>(pr, X0, X1, w, lane, ring_s, bar_s, pol, pre, lens, p);

  // An empty sequence has no tiles: its output rows are zeros (CTAs share the writes).
  const int row_words = p.num_kv_heads * G * kD / 8;  // 16-byte words per sequence
  for (int b = blockIdx.x; b < p.batch; b += p.total_ctas)
    if (pre[b + 1] == pre[b])
      for (int i = tid; i < row_words; i += kThreads)
        reinterpret_cast<uint4*>(p.out + static_cast<size_t>(b) * p.num_kv_heads * G * kD)[i] =
            make_uint4(0u, 0u, 0u, 0u);
  if (!has_tiles) return;  // the whole CTA (no copies were issued): nothing else to do

  // A warp's partial of uf goes to its part of the merge buffer and its partial of ul
  // (always its last segment, when its ring has drained) to its ring's first slot;
  // partials of the units between go to the warp's global slot.  All of them are merged
  // at the CTA's end.
  const int unit_f = uf.b * p.num_kv_heads + uf.h;
  const int unit_l = ul.b * p.num_kv_heads + ul.h;
  auto out_row = [&](int b, int h) {
    return p.out + (static_cast<size_t>(b) * p.num_kv_heads * G + h * G) * kD;
  };
  auto warp_slot = [&](int unit, int ww) {
    return p.part + (static_cast<size_t>(unit + kc) * kWarps + ww) * G * kPartStride;
  };
  float* const rec_f = mbuf;                             // [kWarps][G][kPartStride]
  float* const rec_l = reinterpret_cast<float*>(ring);   // warp ww's: + ww*kStages*kSlot

  int consumed = 0;   // tiles of this warp consumed (tile t uses slot t % kStages)
  bool dead = false;  // a bounded wait gave up: stop touching the ring
  // uf's and ul's q rows: every warp rotates and slices its share of the queries.
  if (!mbar_wait_bounded(qbar_cta, 0u, kWaitLimitNs)) dead = true;
  if (!dead)
    for (int t = 0; t < (two_edges ? 2 : 1); t++)
      prep_q<G, kWarps, FP4>(qraw_all + (kWarps + t) * G * kD * 2, frag_all + (kWarps + t) * kFragWords,
                             sf_all + (kWarps + t) * 8, lane, p, w);
  if (dead && lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);
  __syncthreads();
  State<G> st;
  state_reset<G>(st);
  typename QF<G, FP4>::type qf;
  constexpr int NQ = QFrag<G>::NQ;
  while (x < X1) {
    const int seg_end = min(X1, cu.U + cu.n);
    const int nt = (seg_end - x + kWarps - 1) / kWarps;
    const int x_next = x + kWarps * nt;
    const bool has_next = x_next < X1;
    Unit nu = cu;
    if (has_next) unit_of_tile(nu, x_next, pre, lens, p);
    // q of this unit: rotate and slice into the warp's fragment table; then fetch the
    // next unit's rows into the freed buffer.
    const int table = is_uf(cu) ? kWarps : (is_ul(cu) ? kWarps + 1 : -1);
    if (table >= 0) {
      qfrag_get<G>(qf, frag_all + table * kFragWords, sf_all + table * 8, lane);
    } else {
      if (!dead) {
        if (mbar_wait_bounded(qbar, static_cast<uint32_t>(q_done & 1), kWaitLimitNs)) q_done++;
        else dead = true;
      }
      if (!dead) prep_q<G, 1, FP4>(qraw, frag, sf, lane, p);
      qfrag_get<G>(qf, frag, sf, lane);
    }
    if (has_next && !dead && !is_ul(nu)) q_fetch(nu);
    state_reset<G>(st);
    // Fused append: the warp holding the unit's last tile rotates, quantises and stores the
    // unit's new token, and patches it into that tile's slot once the slot has landed.
    bool new_ok = false;
    if constexpr (FUSED) {
      const int xl = x + kWarps * (nt - 1);  // this warp's last tile of the unit
      uint8_t* patch = reinterpret_cast<uint8_t*>(frag);  // free until the next unit's q
      if (xl == cu.U + cu.n - 1 && !dead) {
        if (!(pre_quantised && x == X0 + w)) {
          const size_t row = (static_cast<size_t>(cu.b) * p.num_kv_heads + cu.h) * kD;
          fused_quantise<FP4>(load_new_row(p.k_new + row, lane), load_new_row(p.v_new + row, lane), lane,
                              patch, p);
        }
        new_ok = fused_store<FP4>(cu.b, cu.h, lane, patch, p);
        if (lane == 0)
          *reinterpret_cast<int*>(patch + PatchLayout<FP4>::kJ) = cu.L - 1 - (xl - cu.U) * kTileTokens;
        __syncwarp();
      }
    }

    auto ntok_of = [&](int xx) { return min(kTileTokens, cu.L - (xx - cu.U) * kTileTokens); };
    // Release a consumed slot and refill it with the warp's tile kStages ahead.
    auto refill = [&]() {
      __syncwarp();
      if (pr.t < pr.nT) {
        fence_proxy_async_smem();
        producer_issue<SEFF, FP4>(pr, X0, X1, w, lane, ring_s, bar_s, pol, pre, lens, p);
      }
    };
    float sc[2][NQ][2];
    int slot_i = consumed % kStages;
    uint32_t parity = static_cast<uint32_t>((consumed / kStages) & 1);
    if (!dead) {
      if (!mbar_wait_bounded(bar_s + 8 * slot_i, parity, kWaitLimitNs)) {
        dead = true;
      } else {
        if constexpr (FUSED) {
          if (new_ok && nt == 1)
            patch_slot<SEFF, FP4>(ring_w + slot_i * kSlot, lane, reinterpret_cast<const uint8_t*>(frag));
        }
        tile_qk_any<G, SEFF>(qf, ring_p + slot_i * kSlot, ntok_of(x), lane, sc);
        float alpha[NQ];
        if (tile_softmax_stats<G>(st, sc, alpha)) tile_rescale<G>(st, alpha);
      }
    }
    // Steady state: a next tile of the unit always exists.  The QK^T and softmax statistics
    // of the next tile are computed next to the PV of the current one; only the rescale
    // of o' has to follow that PV.
    for (int i = 0; i + 1 < nt && !dead; i++) {
      const int xi = x + kWarps * i;
      const int cur = slot_i;
      const int nslot = cur + 1 == kStages ? 0 : cur + 1;
      const uint32_t npar = cur + 1 == kStages ? parity ^ 1u : parity;
      if (!mbar_wait_bounded(bar_s + 8 * nslot, npar, kWaitLimitNs)) {
        dead = true;
        break;
      }
      float sn[2][NQ][2], alpha[NQ];
      if constexpr (FUSED) {
        if (new_ok && i + 2 == nt)
          patch_slot<SEFF, FP4>(ring_w + nslot * kSlot, lane, reinterpret_cast<const uint8_t*>(frag));
      }
      tile_qk_any<G, SEFF>(qf, ring_p + nslot * kSlot, ntok_of(xi + kWarps), lane, sn);
      const bool rescale = tile_softmax_stats<G>(st, sn, alpha);
      tile_pv_any<G, SEFF, FP4>(st, ring_p + cur * kSlot, ntok_of(xi), lane, sc);
      consumed++;
      slot_i = nslot;
      parity = npar;
      refill();
      if (rescale) tile_rescale<G>(st, alpha);
#pragma unroll
      for (int j = 0; j < 2; j++)
#pragma unroll
        for (int qq = 0; qq < NQ; qq++)
#pragma unroll
          for (int r = 0; r < 2; r++) sc[j][qq][r] = sn[j][qq][r];
    }
    if (!dead) {  // last tile of the unit for this warp
      tile_pv_any<G, SEFF, FP4>(st, ring_p + slot_i * kSlot, ntok_of(x + kWarps * (nt - 1)), lane, sc);
      consumed++;
      refill();
    }
    if (dead && lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);

    const int unit = cu.b * p.num_kv_heads + cu.h;
    if (cu.n == 1) {
      // This warp is the unit's only contributor: finish it now (the fragment table is
      // free until the next unit's q is prepared).
      finish_from_state<G>(st, reinterpret_cast<float*>(frag), out_row(cu.b, cu.h), lane, p);
    } else if (unit == unit_f) {
      state_write<G>(st, rec_f + w * G * kPartStride, lane);
    } else if (unit == unit_l) {
      state_write<G>(st, rec_l + w * (kStages * kSlot / 4), lane);
    } else {
      state_write<G>(st, warp_slot(unit, w), lane);
    }
    x = x_next;
    cu = nu;
  }

  // ---- CTA end: every partial of the range is written (shared or global memory).
  __syncthreads();
  // The (one or two) edge units: merge the warps' partials from shared memory, queries
  // split over the warps.  A unit inside the range is finished here; a shared one leaves
  // one record per CTA at the CTA's slot (warp slot 0).
  const int nedge = unit_l == unit_f ? 1 : 2;
  bool shared_edge[2] = {false, false};
#pragma unroll
  for (int e = 0; e < 2; e++) {
    if (e >= nedge) break;
    const Unit& u = e == 0 ? uf : ul;
    const int unit = e == 0 ? unit_f : unit_l;
    const int a = max(X0, u.U), c = min(X1, u.U + u.n) - a;  // this CTA's tiles of u
    shared_edge[e] = !(u.U >= X0 && u.U + u.n <= X1);
    if (u.n == 1) continue;  // already finished by its warp
    float* base = e == 0 ? rec_f : rec_l;
    const int wstride = e == 0 ? G * kPartStride : kStages * kSlot / 4;
    auto rec = [&](int j) -> const float* { return base + ((a - X0 + j) & (kWarps - 1)) * wstride; };
    merge_few<G, kWarps, false, kWarps>(min(kWarps, c), rec, w, out_row(u.b, u.h),
                                        shared_edge[e] ? warp_slot(unit, 0) : nullptr, lane, p);
  }
  // Units between the edges (wholly inside the range, at least two tiles): their warps'
  // records are in global memory; warp w merges every kWarps-th of them.
  if (nedge == 2) {
    Unit u = uf;
    unit_next(u, pre, lens, p);
    for (int i = 0; !(u.b == ul.b && u.h == ul.h); i++, unit_next(u, pre, lens, p)) {
      if ((i & (kWarps - 1)) != w || u.n == 1) continue;
      const int unit = u.b * p.num_kv_heads + u.h;
      auto rec = [&](int j) -> const float* { return warp_slot(unit, (u.U - X0 + j) & (kWarps - 1)); };
      merge_few<G, 1, true, kWarps>(min(kWarps, u.n), rec, 0, out_row(u.b, u.h), nullptr, lane, p);
    }
  }
  // Shared edge units: publish this CTA's record (a CTA barrier, then one acquire-release
  // arrival per unit); the last of the unit's CTAs merges.
  if (shared_edge[0] || shared_edge[1]) {
    __syncthreads();
    if (lane == 0 && w < nedge && shared_edge[w]) {
      const Unit& u = w == 0 ? uf : ul;
      const int unit = w == 0 ? unit_f : unit_l;
      const int ncta = (u.U + u.n - 1) / chunk - u.U / chunk + 1;
      const int old = atom_add_acq_rel_gpu(p.counters + unit, 1);
      const int last = old == ncta - 1;
      if (last) p.counters[unit] = 0;  // ready for the next call
      last_flag_e[w] = last;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 2; e++) {
      if (e >= nedge || !shared_edge[e] || !last_flag_e[e]) continue;
      const Unit& u = e == 0 ? uf : ul;
      const int unit = e == 0 ? unit_f : unit_l;
      const int k0 = u.U / chunk, ncta = (u.U + u.n - 1) / chunk - k0 + 1;
      auto rec = [&](int j) -> const float* {
        return p.part + (static_cast<size_t>(unit + k0 + j) * kWarps) * G * kPartStride;
      };
      if (ncta <= 8)
        merge_few<G, kWarps, true, 8>(ncta, rec, w, out_row(u.b, u.h), nullptr, lane, p);
      else
        merge_records<G, kWarps, true>(ncta, rec, w, out_row(u.b, u.h), nullptr, lane, p);
    }
  }

  if (dead) {
    // Let copies still in flight land before the CTA's shared memory is released.
    for (int j = consumed; j < pr.t; j++)
      mbar_wait_bounded(bar_s + 8 * (j % kStages), static_cast<uint32_t>((j / kStages) & 1),
                        kWaitLimitNs);
    for (; q_done < q_issued; q_done++)
      mbar_wait_bounded(qbar, static_cast<uint32_t>(q_done & 1), kWaitLimitNs);
    mbar_wait_bounded(qbar_cta, 0u, kWaitLimitNs);
  }
}

template <int G, int SEFF>
void* kernel_ptr(bool fused, bool fp4) {
  if (fp4)
    return fused ? reinterpret_cast<void*>(&decode_kernel<G, SEFF, true, true>)
                 : reinterpret_cast<void*>(&decode_kernel<G, SEFF, false, true>);
  return fused ? reinterpret_cast<void*>(&decode_kernel<G, SEFF, true, false>)
               : reinterpret_cast<void*>(&decode_kernel<G, SEFF, false, false>);
}

void* pick_kernel(int group, int seff, bool fused, bool fp4) {
#define KVQ_PICK(GG)                                         \
  if (group == GG) {                                         \
    if (seff == 16) return kernel_ptr<GG, 16>(fused, fp4);   \
    if (seff == 32) return kernel_ptr<GG, 32>(fused, fp4);   \
  }
  KVQ_PICK(1)
  KVQ_PICK(2)
  KVQ_PICK(4)
  KVQ_PICK(8)
#undef KVQ_PICK
  return nullptr;
}

size_t smem_bytes(int group, int max_batch, bool fp4) {
  size_t s = static_cast<size_t>(kWarps) * kStages * slot_bytes(fp4);  // rings
  s += static_cast<size_t>(kWarps + 2) * group * kD * 2;             // raw q rows
  s += sizeof(uint32_t) * (kWarps + 2) * frag_words(group, fp4);     // q fragment tables
  s += sizeof(float) * (kWarps + 2) * 8;                             // M factors
  s += sizeof(float) * kWarps * group * kPartStride;                 // CTA merge buffer
  s += sizeof(uint64_t) * (kWarps * (kStages + 1) + 1);              // mbarriers
  s += static_cast<size_t>(2 * max_batch + 1) * sizeof(int32_t);     // prefix, lengths
  s += 128;                                                          // alignment slack
  return (s + 15) & ~static_cast<size_t>(15);
}

}  // namespace

int plan_decode(int group, int page_size, int max_batch, int num_sms, int fp4, DecodeLaunch* out) {
  const int seff = page_size < kTileTokens ? page_size : kTileTokens;
  const size_t smem = smem_bytes(group, max_batch, fp4 != 0);
  // The dynamic shared memory cap of the variants is set to the most any call of this
  // library uses (max_batch 4096), so plans made for several caches never shrink it
  // under one another; the grid is the smaller occupancy of the variants (plain and
  // fused).
  const size_t cap_bytes = smem_bytes(group, 4096, fp4 != 0);
  int occ = 3;
  for (int fused = 0; fused < 2; fused++) {
    void* fn = pick_kernel(group, seff, fused != 0, fp4 != 0);
    if (!fn) return -1;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(cap_bytes)) != cudaSuccess)
      return -2;
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, fn, kThreads, smem) != cudaSuccess)
      return -2;
    if (o < occ) occ = o;
  }
  if (occ < 1) return -1;
  out->grid = num_sms * occ;
  out->smem = smem;
  return 0;
}

int launch_decode(const DecodeParams& p, const DecodeLaunch& L, cudaStream_t stream) {
  const int seff = p.page_size < kTileTokens ? p.page_size : kTileTokens;
  void* fn = pick_kernel(p.group, seff, p.k_new != nullptr, p.fp4 != 0);
  if (!fn) return -1;
  DecodeParams q = p;
  q.total_ctas = L.grid;
  void* args[] = {&q};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.smem;
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

// append_kernel.cu -- fused block-diagonal Hadamard rotation + token-wise INT4
// quantisation + paged append, for sm_100a.
//
// Method: "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化"
// (youngju.dev), sections "回転のトリック — ブロック対角アダマール" (rotation inside
// blocks of channels), "素朴なINT4はなぜ崩れるのか" (one scale per token, quantised
// as the token is produced) and "システムこそが設計である — 融合カーネル" (one fused
// kernel that rotates, quantises and appends into paged KV blocks without revisiting
// past tokens).
//
// Work decomposition.  Every warp runs its own pipeline: a warp stage is 8 consecutive
// (token, KV head) pairs, their K rows (2 KB, contiguous in the token-packed input) and V
// rows (2 KB), brought into a ring of 3 shared-memory slots by two 1-D bulk copies (TMA
// engine, no multicast) that complete on the slot's mbarrier.  Warps take warp stages
// gw, gw + W, ... (gw = the global warp index, W = all warps of the persistent grid) and
// never wait for one another, so their serial parts (the row's scale, the stores) spread
// out in time; no register holds prefetched data.  Two lanes handle one row (the K or V
// row of one pair, 128 fp16 channels): lane l holds channels [64l, 64l + 64) as 8 chunks
// of 8 channels.
//
// Bank-conflict-free reads.  A lane reads its chunks in the order c = t ^ rho (t = 0..7,
// rho = lane & 7): the 8 lanes of a quarter warp then touch 8 different 16-byte bank
// groups.  Register slot t holds chunk t ^ rho, so the butterfly stages that pair chunks
// (h = 8, 16, 32: chunk bits 0-2) pair slots t and t ^ k as well; whether slot t holds the
// lower or the upper chunk of the pair depends on rho, and each output is one fma with a
// +-1 multiplier (fma(a, 1, c) = a + c and fma(c, -1, a) = a - c, rounded once: the IEEE
// sum and difference).  Stages h = 1, 2, 4 are inside a chunk.  Only b = 128 has a stage
// across the lane pair (h = 64): lane 1's slot t ^ 1 holds the partner of lane 0's slot t
// (their rho differ in bit 0); after one exchange lane 0 keeps the sums (channels
// [0, 64)) and lane 1 the differences (channels [64, 128)), in the same slot order.
//
// Stages run in the fixed order h = 1, 2, ..., b/2, each pair (i, i + h) with bit h of i
// clear becoming (a + c, a - c) as one IEEE fp32 add and one subtract, then one multiply
// by the fp32 constant nearest 1/sqrt(b): rotated values are bit-exact with any
// implementation of that fixed-order butterfly.  Pairs of channels go through the packed
// fp32x2 arithmetic of sm_100 (each half is still one IEEE operation) held in 64-bit
// registers; fp16 -> fp32 conversion rides in the first stage's mixed-precision adds.
//
// Quantisation: m = max |y| (lane-pair shuffle), s = fp16_rn(m / 7) (IEEE division, once
// per row).  Codes are round-half-even of y / s, clamped to [-8, 7], computed without
// dividing: a fast multiply-by-reciprocal path, and an exact half-point comparison for
// groups with a near-tie (see quantise()); codes stay bit-exact with division by the
// stored fp16 scale.  Codes are packed two per byte (low nibble = even channel).  A
// lane's 8 code words (one per chunk, in slot order) go through a per-warp staging area
// in shared memory, written at their chunk's place and read back in channel order, so
// that the row's 64 code bytes leave as two 16-byte stores per lane (one L2 request per
// row and store); lane 0 of the row stores the scale.
//
// NVFP4 rows ("BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号" (sns.style), sections
// "背景と概要", "深掘り分析": 4-bit microscaling elements with E4M3 block scales): after
// the same rotation, each block of 16 channels -- slots t and t ^ 1 of a lane, since the
// rotation of the read order keeps chunk pairs together -- gets s = E4M3(fl(max|y| / 6))
// (round to nearest even, saturated at 448) and codes E2M1(fl(y * fl(1/s))) (nearest
// even, saturated at 6, sign kept), both by the hardware conversions cvt.rn.satfinite;
// all codes 0 when s == 0.  A lane's 4 scale bytes are stored as one word.
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kD = 128;
constexpr int kPairs = 8;                      // (token, KV head) pairs per warp stage
constexpr int kWarps = 8;                      // warps per CTA
constexpr int kThreads = 32 * kWarps;
constexpr int kHalfBytes = kPairs * kD * 2;    // one tensor's rows of a warp stage: 2 KB
constexpr int kSlotBytes = 2 * kHalfBytes;     // K rows, then V rows
constexpr int kStages = 3;                     // ring slots per warp
constexpr int kStgStride = 80;                 // staging bytes per row (64 used)
// A warp's region: ring slots | staging lines | sequence cursors (16 B per pair slot) |
// barriers, rounded to 128 bytes so that every region (and so every copy destination)
// stays 16-byte aligned.
constexpr int kCursorBytes = 16 * kPairs;
constexpr int kWarpBytes =
    (kStages * kSlotBytes + 2 * kPairs * kStgStride + kCursorBytes + 8 * kStages + 127) / 128 * 128;
constexpr int kSmemBytes = kWarps * kWarpBytes;
constexpr int kCtasPerSm = 2;
static_assert(kCtasPerSm * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM must fit");
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s

// Two fp32 values in one 64-bit register (low half = the even channel).
typedef unsigned long long f2;

__device__ __forceinline__ f2 pk(float a, float b) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk(f2 v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
  f2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2 sub2(f2 a, f2 b) {
  f2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// a * b + c per half, one rounding each.
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// fp16 bits -> fp32, exact (h + -0.0 keeps signed zeros).
__device__ __forceinline__ float cvt_f16(uint32_t h) {
  float d;
  asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(static_cast<uint16_t>(h)), "f"(-0.0f));
  return d;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Issue the two bulk copies of warp stage j (pairs [8j, 8j + n)) into the slot at dst.
__device__ __forceinline__ void issue_stage(const AppendParams& p, int j, int npairs,
                                            uint32_t dst, uint32_t bar, uint64_t pol) {
  const int g0 = j * kPairs;
  const int left = npairs - g0;
  const uint32_t bytes = static_cast<uint32_t>(left < kPairs ? left : kPairs) * (kD * 2);
  mbar_arrive_expect_tx(bar, 2 * bytes);
  bulk_copy_g2s(dst, p.k + static_cast<size_t>(g0) * kD, bytes, bar, pol);
  bulk_copy_g2s(dst + kHalfBytes, p.v + static_cast<size_t>(g0) * kD, bytes, bar, pol);
}

// Where pair gp goes: its sequence b (the b with cu[b] <= t < cu[b+1]), position pos =
// seq_lens[b] + t - cu[b], the raw page-table entry of page pos / S (checked at use, so
// that the load is in flight meanwhile) and the slot pos % S, or slot -1 for a position
// outside the page table.
struct Dest {
  int page;
  int slot;
  int h;
};

// The sequence of a pair slot's current token, kept in shared memory across the warp's
// stages (whose tokens only increase) as {b, cu_lo, cu_hi, sl}: [cu_lo, cu_hi) = the
// sequence's tokens in the call, sl = its length before the call.  A token outside the
// range moves the cursor by a binary search over cu_new_tokens; a token inside it needs no
// global load.  The four lanes of a pair read and write the same entry with the same
// values; the warp syncs between stages.
__device__ __forceinline__ Dest pair_dest(const AppendParams& p, int gp, uint32_t cursor) {
  Dest d;
  // t = gp / num_kv_heads by the host's multiplier (gp < 2^31); pos / S and pos % S by
  // the power-of-two page size.
  const int t = static_cast<int>(__umulhi(static_cast<uint32_t>(gp) << 1, p.heads_magic) >> p.heads_shift);
  d.h = gp - t * p.num_kv_heads;
  uint4 sc = lds_128(cursor);  // x = b, y = cu_lo, z = cu_hi, w = sl
  if (t < static_cast<int>(sc.y) || t >= static_cast<int>(sc.z)) {
    int lo = 0, hi = p.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(p.cu_new_tokens + mid) <= t) lo = mid; else hi = mid;
    }
    sc = make_uint4(static_cast<uint32_t>(lo), static_cast<uint32_t>(__ldg(p.cu_new_tokens + lo)),
                    static_cast<uint32_t>(__ldg(p.cu_new_tokens + lo + 1)),
                    static_cast<uint32_t>(__ldg(p.seq_lens + lo)));
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(cursor), "r"(sc.x), "r"(sc.y), "r"(sc.z),
                 "r"(sc.w)
                 : "memory");
  }
  const int b = static_cast<int>(sc.x);
  const int pos = static_cast<int>(sc.w) + (t - static_cast<int>(sc.y));
  const int lp = pos >= 0 ? pos >> p.page_shift : 0;
  if (pos < 0 || lp >= p.max_pages_per_seq) {
    d.page = -1;
    d.slot = -1;
  } else {
    d.page = __ldg(p.page_table + static_cast<size_t>(b) * p.max_pages_per_seq + lp);
    d.slot = pos & (p.page_size - 1);
  }
  return d;
}

// The butterfly without its final scale: x = z, the rotated row being y = fl(c_b * z),
// which quantise() applies where it needs y itself.  raw[t] = chunk t ^ rho of this lane's
// half row (4 words = 8 fp16 channels); x[4t + e] = channels 2e, 2e + 1 of that chunk.
template <int BLOCK>
__device__ __forceinline__ void rotate_row(const uint4 (&raw)[8], int rho, int l, unsigned pmask,
                                           f2 (&x)[32]) {
#pragma unroll
  for (int t = 0; t < 8; t++) {
    const uint32_t w[4] = {raw[t].x, raw[t].y, raw[t].z, raw[t].w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
      if constexpr (BLOCK == 1) {
        // b = 1 (plain INT4): the transform of size 1 is the identity and c_b = 1.
        x[4 * t + e] = pk(cvt_f16(w[e] & 0xffffu), cvt_f16(w[e] >> 16));
      } else {
        // Stage h = 1 fused with the conversion: (a, c) -> (a + c, a - c).
        const float c = cvt_f16(w[e] >> 16);
        const uint16_t lo = static_cast<uint16_t>(w[e] & 0xffffu);
        float s, d;
        asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(s) : "h"(lo), "f"(c));
        asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(lo), "f"(c));
        x[4 * t + e] = pk(s, d);
      }
    }
  }
  if constexpr (BLOCK > 1) {
    // Stages h = 2 (pair index e <-> e + 1) and h = 4 (e <-> e + 2) inside each chunk.
#pragma unroll
    for (int t = 0; t < 8; t++)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const f2 a = x[4 * t + e], c = x[4 * t + e + 1];
        x[4 * t + e] = add2(a, c);
        x[4 * t + e + 1] = sub2(a, c);
      }
#pragma unroll
    for (int t = 0; t < 8; t++)
#pragma unroll
      for (int e = 0; e < 2; e++) {
        const f2 a = x[4 * t + e], c = x[4 * t + e + 2];
        x[4 * t + e] = add2(a, c);
        x[4 * t + e + 2] = sub2(a, c);
      }
    // Stages h = 8, 16, 32: chunk bit k, slots t and t ^ (1 << k).  With bit k of rho
    // clear slot t holds the lower chunk: (t, u) <- (t + u, t - u); set: (u, t) <- (u + t,
    // u - t).  Both as fma(own, sg, other), sg = +-1.
#pragma unroll
    for (int k = 0; k < 3; k++) {
      if ((8 << k) < BLOCK) {
        const float sg = ((rho >> k) & 1) ? -1.0f : 1.0f;
        const f2 SG = pk(sg, sg), NSG = pk(-sg, -sg);
#pragma unroll
        for (int t = 0; t < 8; t++) {
          if (t & (1 << k)) continue;
          const int u = t | (1 << k);
#pragma unroll
          for (int e = 0; e < 4; e++) {
            const f2 a = x[4 * t + e], c = x[4 * u + e];
            x[4 * t + e] = fma2(a, SG, c);
            x[4 * u + e] = fma2(c, NSG, a);
          }
        }
      }
    }
    if constexpr (BLOCK == 128) {
      // Stage h = 64 across the lane pair.  Lane 0's slot t and lane 1's slot t ^ 1 hold
      // the same chunk of their halves (rho differs in bit 0 between them), so every lane
      // receives its partner's slot t ^ 1 for its slot t.  Lane 0 (the lower channel)
      // keeps own + other, lane 1 (the upper) other - own: fma(own, +-1, other).
      const float sg = l ? -1.0f : 1.0f;
      const f2 SG = pk(sg, sg);
#pragma unroll
      for (int t = 0; t < 8; t += 2)
#pragma unroll
        for (int e = 0; e < 4; e++) {
          float a0, a1, c0, c1;
          upk(x[4 * t + e], a0, a1);
          upk(x[4 * (t + 1) + e], c0, c1);
          const f2 ra = pk(__shfl_xor_sync(pmask, c0, 1), __shfl_xor_sync(pmask, c1, 1));
          const f2 rc = pk(__shfl_xor_sync(pmask, a0, 1), __shfl_xor_sync(pmask, a1, 1));
          x[4 * t + e] = fma2(x[4 * t + e], SG, ra);
          x[4 * (t + 1) + e] = fma2(x[4 * (t + 1) + e], SG, rc);
        }
    }
  }
}

// The 8 codes of one chunk from their magic-rounded values (code = low nibble of the
// bits), packed low nibble = even channel.
__device__ __forceinline__ uint32_t pack_chunk(const f2 (&m)[4]) {
  float v[8];
#pragma unroll
  for (int e = 0; e < 4; e++) upk(m[e], v[2 * e], v[2 * e + 1]);
  const uint32_t ev = prmt(prmt(__float_as_uint(v[0]), __float_as_uint(v[2]), 0x0040u),
                           prmt(__float_as_uint(v[4]), __float_as_uint(v[6]), 0x0040u), 0x5410u);
  const uint32_t od = prmt(prmt(__float_as_uint(v[1]), __float_as_uint(v[3]), 0x0040u),
                           prmt(__float_as_uint(v[5]), __float_as_uint(v[7]), 0x0040u), 0x5410u);
  uint32_t r;
  // (ev & 0x0F0F0F0F) | ((od << 4) & 0xF0F0F0F0)
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(r) : "r"(ev), "r"(od << 4), "r"(0x0F0F0F0Fu));
  return r;
}

// Quantise this lane's 64 values of a row; q[t] = packed codes of slot t's chunk.
// Returns the fp16 scale bits (identical on both lanes of the row).
//
// Codes are round-half-even of y / s with s the stored fp16 scale.  Fast path (a normal,
// unsaturated s, so |y/s| <= 7.004): t = z * fl(c_b * fl(1/s)) (exact product) is within
// 4 roundings (< 2^-19) of y / s; fma(z, r_z, 1.5 * 2^23) rounds it to the nearest integer
// (ties to even) in one step, and fma(z, r_z, -rint) gives t - rint with one rounding, so
// the result is exact unless the fraction is within 2^-19 of one half.  A chunk with such
// a near-tie -- frequent for rows that are not rotated, whose fp16 values meet exact ties
// -- and every chunk when s is subnormal or saturated is recomputed exactly without
// dividing: k = floor(y*r) is within one of the true floor, and (k + 1/2)*s is exact in
// fp32 (an fp16 scale times a number of 5 bits), so comparing y with it chooses between k
// and k + 1, an exact tie going to the even one.  (If y*r fell on the wrong side of an
// integer n, y/s is within 2^-16 of n and both candidates' half points place it at n.)
// Codes are clamped to [-8, 7].
__device__ __forceinline__ uint16_t quantise(const f2 (&x)[32], float cb, unsigned pmask,
                                             uint32_t (&q)[8]) {
  // m = max |y| = fl(c_b * max |z|): rounding is monotonic, so scaling after the max gives
  // the max of the scaled values.
  float cm[8];  // per chunk, then a tree: short dependency chains
#pragma unroll
  for (int t = 0; t < 8; t++) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 4; e++) upk(x[4 * t + e], v[2 * e], v[2 * e + 1]);
    cm[t] = max3(max3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])),
                 max3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7])));
  }
  float zmax = max3(max3(cm[0], cm[1], cm[2]), max3(cm[3], cm[4], cm[5]), fmaxf(cm[6], cm[7]));
  zmax = fmaxf(zmax, __shfl_xor_sync(pmask, zmax, 1));
  const float m = __fmul_rn(cb, zmax);
  const float s32 = __fdiv_rn(m, 7.0f);
  const bool sat = s32 > 65504.0f;
  const __half sh = sat ? __ushort_as_half(0x7BFF) : __float2half_rn(s32);
  const float s = __half2float(sh);
  if (s == 0.0f) {  // an all-zero row (or a scale that underflows): every code is 0
#pragma unroll
    for (int t = 0; t < 8; t++) q[t] = 0u;
    return __half_as_ushort(sh);
  }
  const bool normal = !sat && s >= 6.103515625e-05f;
  const float r = __frcp_rn(s);
  const float rz = __fmul_rn(cb, r);
  const float hs = 0.5f * s;
  const f2 MM = pk(kMagic, kMagic);
  const f2 RZ = pk(rz, rz);
  // Fast path for 4 chunks at a time, without branches; chunks with a near-tie are marked
  // and then recomputed exactly (rare for rotated rows).
#pragma unroll
  for (int g = 0; g < 8; g += 4) {
    uint32_t redo = normal ? 0u : 0xFFu;
#pragma unroll
    for (int t = g; t < g + 4; t++) {
      f2 mg[4];
      float d[8];
#pragma unroll
      for (int e = 0; e < 4; e++) {
        mg[e] = fma2(x[4 * t + e], RZ, MM);   // 1.5*2^23 + rint(t)
        const f2 nr = sub2(MM, mg[e]);        // -rint(t), exactly
        upk(fma2(x[4 * t + e], RZ, nr), d[2 * e], d[2 * e + 1]);  // t - rint(t)
      }
      const float dmax = max3(max3(fabsf(d[0]), fabsf(d[1]), fabsf(d[2])),
                              max3(fabsf(d[3]), fabsf(d[4]), fabsf(d[5])), fmaxf(fabsf(d[6]), fabsf(d[7])));
      if (!(dmax < 0.5f - 0x1p-19f)) redo |= 1u << t;
      q[t] = pack_chunk(mg);
    }
    if (redo) {
#pragma unroll
      for (int t = g; t < g + 4; t++) {
        if (!((redo >> t) & 1u)) continue;
        f2 mg[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
          float z[2], o[2];
          upk(x[4 * t + e], z[0], z[1]);
#pragma unroll
          for (int i = 0; i < 2; i++) {
            const float y = __fmul_rn(z[i], cb);  // the rotated value
            const float k = floorf(__fmul_rn(y, r));
            const float h = __fmaf_rn(k, s, hs);  // (k + 1/2) * s, exact
            const bool odd = (__float_as_uint(__fadd_rn(k, kMagic)) & 1u) != 0u;
            const bool up = y > h || (y == h && odd);
            const float c = fminf(fmaxf(up ? k + 1.0f : k, -8.0f), 7.0f);
            o[i] = __fadd_rn(c, kMagic);
          }
          mg[e] = pk(o[0], o[1]);
        }
        q[t] = pack_chunk(mg);
      }
    }
  }
  return __half_as_ushort(sh);
}

// Two fp32 values -> one byte of E2M1 codes (lo -> low nibble), nearest even, saturating.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 q;\n\tcvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\tcvt.u32.u8 %0, q;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 values -> two E4M3 bytes (lo -> low byte), nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 bytes (low 16 bits) -> their values (exact).
__device__ __forceinline__ float2 e4m3x2_value(uint32_t b) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(b)));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// NVFP4 quantisation of this lane's 64 values: q[t] = the 4 code bytes of slot t's chunk;
// returns the lane's 4 scale bytes in block order (byte m = block 4l + m of the row).
__device__ __forceinline__ uint32_t quantise_fp4(const f2 (&x)[32], float cb, int rho,
                                                uint32_t (&q)[8]) {
  const f2 CB = pk(cb, cb);
  float sv[4];
  uint32_t sb[4];
#pragma unroll
  for (int u = 0; u < 4; u++) {  // slot pair (2u, 2u + 1) = one block of 16 channels
    float v[16];
#pragma unroll
    for (int e = 0; e < 8; e++) upk(x[8 * u + e], v[2 * e], v[2 * e + 1]);
    const float m8a = max3(max3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])),
                           max3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7])));
    const float m8b = max3(max3(fabsf(v[8]), fabsf(v[9]), fabsf(v[10])),
                           max3(fabsf(v[11]), fabsf(v[12]), fabsf(v[13])), fmaxf(fabsf(v[14]), fabsf(v[15])));
    // max |y| = fl(c_b * max |z|) (rounding is monotonic)
    sv[u] = __fdiv_rn(__fmul_rn(cb, fmaxf(m8a, m8b)), 6.0f);
  }
  const uint32_t s01 = e4m3x2(sv[0], sv[1]), s23 = e4m3x2(sv[2], sv[3]);
  sb[0] = s01 & 0xFFu;
  sb[1] = s01 >> 8;
  sb[2] = s23 & 0xFFu;
  sb[3] = s23 >> 8;
  const float2 f01 = e4m3x2_value(s01), f23 = e4m3x2_value(s23);
  const float sf[4] = {f01.x, f01.y, f23.x, f23.y};
#pragma unroll
  for (int u = 0; u < 4; u++) {
    const float r = sf[u] != 0.0f ? __frcp_rn(sf[u]) : 0.0f;
    const f2 R = pk(r, r);
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const int t = 2 * u + h;
      uint32_t w = 0;
#pragma unroll
      for (int e = 0; e < 4; e++) {
        float a, b;
        upk(mul2(mul2(x[4 * t + e], CB), R), a, b);  // t = fl(fl(z * c_b) * r)
        w |= e2m1x2(a, b) << (8 * e);
      }
      q[t] = sf[u] != 0.0f ? w : 0u;  // a zero scale: every code 0
    }
  }
  // Byte u of the word belongs to block (2u ^ rho) >> 1 = u ^ (rho >> 1) of the lane's half.
  const uint32_t words = sb[0] | (sb[1] << 8) | (sb[2] << 16) | (sb[3] << 24);
  const uint32_t r2 = static_cast<uint32_t>(rho >> 1);
  const uint32_t sel = (0u ^ r2) | ((1u ^ r2) << 4) | ((2u ^ r2) << 8) | ((3u ^ r2) << 12);
  return prmt(words, 0u, sel);
}

template <int BLOCK, bool FP4>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) append_kernel(AppendParams p) {
  // The next kernel may start its own prologue; the pool stores below wait for every
  // earlier kernel (griddep_wait), so they never race with a decode still reading.
  griddep_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  // This warp's ring, staging lines and barriers.
  const uint32_t ring = smem_addr(smem) + w * kWarpBytes;
  const uint32_t stg = ring + kStages * kSlotBytes;
  const uint32_t cursors = stg + 2 * kPairs * kStgStride;
  const uint32_t bar0 = cursors + kCursorBytes;
  const int l = lane & 1, rho = lane & 7;
  const int pr = lane >> 2;         // pair within the warp stage
  const int kv = (lane >> 1) & 1;   // 0 = K row, 1 = V row
  // Shuffles never leave the lane pair of a row, so they name only those two lanes.
  const unsigned pmask = 0x3u << (lane & 30);
  const int npairs = p.total_new_tokens * p.num_kv_heads;  // < 2^31 (host-checked)
  const int nws = (npairs + kPairs - 1) / kPairs;
  const int W = gridDim.x * kWarps;
  const int gw = blockIdx.x * kWarps + w;
  // This row's 80-byte staging line; the lane's half is at +32l.
  const uint32_t stg_row = stg + (lane >> 1) * kStgStride + 32 * l;
  const uint64_t pol = l2_policy_evict_first();

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; s++) mbar_init(bar0 + 8 * s, 1);
    fence_mbar_init();
#pragma unroll
    for (int s = 0; s < kStages; s++) {
      const int j = gw + s * W;
      if (j < nws) issue_stage(p, j, npairs, ring + s * kSlotBytes, bar0 + 8 * s, pol);
    }
  }
  __syncwarp();

  const uint32_t cursor = cursors + 16 * pr;  // this lane's pair slot
  if ((lane & 3) == 0)  // an empty range: the first lookup searches
    asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(cursor), "r"(0u) : "memory");
  __syncwarp();
  Dest dcur = {-1, -1, 0};
  if (gw * kPairs + pr < npairs) dcur = pair_dest(p, gw * kPairs + pr, cursor);
  bool waited = false;
  int s = 0;
  uint32_t phase = 0;
  for (int j = gw; j < nws; j += W) {
    const uint32_t slot = ring + s * kSlotBytes;
    const int gp = j * kPairs + pr;
    const bool active = gp < npairs;
    // The next warp stage's destination: its page-table load is in flight meanwhile.
    Dest dnext = {-1, -1, 0};
    if (j + W < nws && gp + W * kPairs < npairs) dnext = pair_dest(p, gp + W * kPairs, cursor);

    if (!mbar_wait_bounded(bar0 + 8 * s, phase, kWaitLimitNs)) {
      // A copy did not land in time: flag it, let this warp's other copies finish
      // (bounded) so nothing lands in shared memory after the CTA exits, and stop.
      if (lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);
#pragma unroll
      for (int k = 1; k < kStages; k++) {
        const int sk = (s + k) % kStages;
        if (j + k * W < nws)
          mbar_wait_bounded(bar0 + 8 * sk, sk > s ? phase : phase ^ 1u, kWaitLimitNs);
      }
      return;
    }
    uint4 raw[8];
    if (active) {
      const uint32_t row = slot + kv * kHalfBytes + pr * (kD * 2) + l * kD;
#pragma unroll
      for (int t = 0; t < 8; t++) raw[t] = lds_128(row + 16 * (t ^ rho));
    }
    // Every read of this slot is done: it can take warp stage j + kStages * W.
    __syncwarp();
    if (lane == 0 && j + kStages * W < nws) {
      fence_proxy_async_smem();
      issue_stage(p, j + kStages * W, npairs, slot, bar0 + 8 * s, pol);
    }
    if (++s == kStages) {
      s = 0;
      phase ^= 1u;
    }

    if (active) {  // both lanes of a row, and both rows of a pair, take the same branch
      f2 x[32];
      rotate_row<BLOCK>(raw, rho, l, pmask, x);
      uint32_t q[8];
      uint32_t sbits;
      if constexpr (FP4) sbits = quantise_fp4(x, p.cb, rho, q);
      else sbits = quantise(x, p.cb, pmask, q);
      // Slot t's word is word t ^ rho of the lane's half: through the staging line into
      // channel order (the lane reads back only what it wrote).
#pragma unroll
      for (int t = 0; t < 8; t++) sts_32(stg_row + 4 * (t ^ rho), q[t]);
      const uint4 c0 = lds_128(stg_row), c1 = lds_128(stg_row + 16);
      if (!waited) {
        griddep_wait();
        waited = true;
      }
      const bool bad_pos = dcur.slot < 0;
      if (bad_pos || dcur.page < 0 || dcur.page >= p.num_pages) {
        if (l == 0 && kv == 0)
          atomicOr(p.status, bad_pos ? KVQ_DEV_BAD_POS_BIT : KVQ_DEV_BAD_PAGE_BIT);
      } else {
        const int S = p.page_size;
        constexpr int kScaleBytes = FP4 ? kD / 16 : 2;  // per token row
        uint8_t* blk = p.pool_layer + (static_cast<size_t>(dcur.page) * p.num_kv_heads + dcur.h) *
                                          (static_cast<size_t>(S) * (kD + 2 * kScaleBytes));
        uint4* crow = reinterpret_cast<uint4*>(blk + static_cast<size_t>(kv) * S * (kD / 2) +
                                               static_cast<size_t>(dcur.slot) * (kD / 2) + 32 * l);
        crow[0] = c0;
        crow[1] = c1;
        uint8_t* srow = blk + static_cast<size_t>(S) * kD + static_cast<size_t>(kv) * S * kScaleBytes +
                        static_cast<size_t>(dcur.slot) * kScaleBytes;
        if constexpr (FP4) {
          *reinterpret_cast<uint32_t*>(srow + 4 * l) = sbits;
        } else {
          if (l == 0) *reinterpret_cast<uint16_t*>(srow) = static_cast<uint16_t>(sbits);
        }
      }
    }
    dcur = dnext;
  }
}

template <int BLOCK, bool FP4>
int launch_block(const cudaLaunchConfig_t& cfg, const AppendParams& p) {
  // The shared-memory opt-in is an attribute of the function in the current device's
  // context: set it once per device (devices 64 and up set it on every launch).
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -2;
  const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
  if (bit == 0 || (attr_set.load(std::memory_order_acquire) & bit) == 0) {
    if (cudaFuncSetAttribute(append_kernel<BLOCK, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
      return -2;
    attr_set.fetch_or(bit, std::memory_order_release);
  }
  return cudaLaunchKernelEx(&cfg, append_kernel<BLOCK, FP4>, p) == cudaSuccess ? 0 : -2;
}

template <bool FP4>
int launch_format(const cudaLaunchConfig_t& cfg, const AppendParams& p, int block) {
  switch (block) {
    case 1: return launch_block<1, FP4>(cfg, p);
    case 32: return launch_block<32, FP4>(cfg, p);
    case 64: return launch_block<64, FP4>(cfg, p);
    case 128: return launch_block<128, FP4>(cfg, p);
    default: return -1;
  }
}

}  // namespace

int launch_append(const AppendParams& p, int block, int num_sms, cudaStream_t stream) {
  const long long npairs = static_cast<long long>(p.total_new_tokens) * p.num_kv_heads;
  if (npairs == 0) return 0;
  if (npairs > 0x7fffffffLL - (64LL << 20)) return -1;  // int indexing in the kernel
  const long long nws = (npairs + kPairs - 1) / kPairs;
  // One wave of persistent CTAs, or fewer for a small call.
  const long long full = static_cast<long long>(kCtasPerSm) * num_sms;
  const long long need = (nws + kWarps - 1) / kWarps;
  const long long grid = need < full ? need : full;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return p.fp4 ? launch_format<true>(cfg, p, block) : launch_format<false>(cfg, p, block);
}

}  // namespace kvq

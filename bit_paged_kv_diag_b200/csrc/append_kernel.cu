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
// Work decomposition.  Two lanes handle one row (the K row or the V row of one
// (token, KV head) pair, 128 fp16 channels); a warp handles the K and V rows of 8 pairs.
// Lane l of a row holds the 16-channel chunks 2j + l (j = 0..3), read with 256-bit loads:
// channel index bits 0-3 and 5-6 are inside the lane and bit 4 is across the lane pair.
// So the butterfly stages h = 1, 2, 4, 8, 32, 64 are register-only and stage h = 16 is one
// warp shuffle.  Stages run in the fixed order h = 1, 2, ..., b/2, each pair (i, i+h) with
// bit h of i clear becoming (a + c, a - c) as one IEEE fp32 add and one subtract, then one
// multiply by the fp32 constant nearest 1/sqrt(b): rotated values are bit-exact with any
// implementation of that fixed-order butterfly.  Pairs of channels go through the packed
// fp32x2 add/sub/mul of sm_100 (each lane of the pair is still one IEEE operation), and
// fp16 -> fp32 conversion rides in the first stage's mixed-precision adds.
//
// Quantisation: m = max |y| (lane-pair shuffle), s = fp16_rn(m / 7) (IEEE division, once
// per row).  Codes are round-half-even of y / s, clamped to [-8, 7], computed without
// dividing: a fast multiply-by-reciprocal path, and an exact half-point comparison for
// groups with a near-tie (see quantise()); codes stay bit-exact with division by the
// stored fp16 scale.  Codes are packed two per byte (low nibble = even channel) and
// written with 64-bit stores; lane 0 of the row stores the fp16 scale.
//
// The CTAs are persistent (one wave, two per SM): each takes row blocks i, i + grid, ...
// and issues the loads of its next rows before computing the current ones.
#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kD = 128;
constexpr int kRowsPerBlock = 128;           // rows (K or V) per CTA
constexpr int kThreads = kRowsPerBlock * 2;  // 2 lanes per row
constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23

__device__ __forceinline__ float cvt_f16(uint16_t h) {
  // Exact fp16 -> fp32 through the mixed-precision add (h + -0.0 keeps signed zeros).
  float d;
  asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(h), "f"(-0.0f));
  return d;
}

// Butterfly on two pairs at once: (a0,a1),(c0,c1) -> (a+c, a-c) per lane, IEEE fp32.
__device__ __forceinline__ void bfly2(float& a0, float& a1, float& c0, float& c1) {
  asm("{\n\t.reg .b64 pa, pc, ps, pd;\n\t"
      "mov.b64 pa, {%0, %1};\n\tmov.b64 pc, {%2, %3};\n\t"
      "add.rn.f32x2 ps, pa, pc;\n\tsub.rn.f32x2 pd, pa, pc;\n\t"
      "mov.b64 {%0, %1}, ps;\n\tmov.b64 {%2, %3}, pd;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(c0), "+f"(c1));
}

// (x0, x1) <- (x0 * s + o0, x1 * s + o1), one rounding each: with s = +-1 this is the
// IEEE sum or difference of the two operands.
__device__ __forceinline__ void fma2(float& x0, float& x1, float s, float o0, float o1) {
  asm("{\n\t.reg .b64 px, ps, po, pd;\n\t"
      "mov.b64 px, {%0, %1};\n\tmov.b64 ps, {%2, %2};\n\tmov.b64 po, {%3, %4};\n\t"
      "fma.rn.f32x2 pd, px, ps, po;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(s), "f"(o0), "f"(o1));
}

__device__ __forceinline__ void mul2(float& x0, float& x1, float s) {
  asm("{\n\t.reg .b64 px, ps, pd;\n\t"
      "mov.b64 px, {%0, %1};\n\tmov.b64 ps, {%2, %2};\n\t"
      "mul.rn.f32x2 pd, px, ps;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(s));
}

// This lane's half of a row: the 16-channel chunks 2j + l (j = 0..3), 256-bit loads.
__device__ __forceinline__ void load_row(const __half* row, int l, u32x8 (&raw)[4]) {
#pragma unroll
  for (int j = 0; j < 4; j++) raw[j] = ldg_256_stream(row + 16 * (2 * j + l));
}

// x[16j + e] = channel 16(2j + l) + e.  b = 1 (plain INT4): the transform of size 1 is
// the identity and c_b = 1, so the row is only converted.
__device__ __forceinline__ void convert_plain(const u32x8 (&raw)[4], float (&x)[64]) {
#pragma unroll
  for (int j = 0; j < 4; j++)
#pragma unroll
    for (int w = 0; w < 8; w++) {
      x[16 * j + 2 * w] = cvt_f16(static_cast<uint16_t>(raw[j].w[w] & 0xffffu));
      x[16 * j + 2 * w + 1] = cvt_f16(static_cast<uint16_t>(raw[j].w[w] >> 16));
    }
}

// The butterfly without its final scale: x = z, the rotated row being y = fl(c_b * z),
// which quantise() applies where it needs y itself.
template <int BLOCK>
__device__ __forceinline__ void rotate_row(const u32x8 (&raw)[4], int l, unsigned pmask,
                                           float (&x)[64]) {
  if constexpr (BLOCK == 1) {
    convert_plain(raw, x);
    return;
  } else {
  // Stage h = 1 fused with the conversion: (a, c) -> (a + c, a - c).
#pragma unroll
  for (int j = 0; j < 4; j++)
#pragma unroll
    for (int w = 0; w < 8; w++) {
      const uint16_t lo = static_cast<uint16_t>(raw[j].w[w] & 0xffffu);
      const uint16_t hi = static_cast<uint16_t>(raw[j].w[w] >> 16);
      const float c = cvt_f16(hi);
      float s, d;
      asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(s) : "h"(lo), "f"(c));
      asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(lo), "f"(c));
      x[16 * j + 2 * w] = s;
      x[16 * j + 2 * w + 1] = d;
    }
  // In-lane stages h = 2, 4, 8 (bits 1-3 of the chunk-local index).
#pragma unroll
  for (int h = 2; h <= 8; h *= 2)
#pragma unroll
    for (int j = 0; j < 4; j++)
#pragma unroll
      for (int e = 0; e < 16; e += 2)
        if (!(e & h)) bfly2(x[16 * j + e], x[16 * j + e + 1], x[16 * j + e + h], x[16 * j + e + h + 1]);
  // Cross-lane stage h = 16: the lane holding the lower index computes own + other, the
  // upper one other - own (fma with a +-1 multiplier rounds once: bit-identical).
  if (16 < BLOCK) {
    const float sgn = l ? -1.0f : 1.0f;
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
      const float o0 = __shfl_xor_sync(pmask, x[i], 1);
      const float o1 = __shfl_xor_sync(pmask, x[i + 1], 1);
      fma2(x[i], x[i + 1], sgn, o0, o1);
    }
  }
  // In-lane stages h = 32 (chunk j with j ^ 1) and h = 64 (chunk j with j ^ 2).
  if (32 < BLOCK) {
#pragma unroll
    for (int j = 0; j < 4; j += 2)
#pragma unroll
      for (int e = 0; e < 16; e += 2)
        bfly2(x[16 * j + e], x[16 * j + e + 1], x[16 * (j + 1) + e], x[16 * (j + 1) + e + 1]);
  }
  if (64 < BLOCK) {
#pragma unroll
    for (int j = 0; j < 2; j++)
#pragma unroll
      for (int e = 0; e < 16; e += 2)
        bfly2(x[16 * j + e], x[16 * j + e + 1], x[16 * (j + 2) + e], x[16 * (j + 2) + e + 1]);
  }
  }
}

// Codes of 8 channels from their magic-rounded sums (low nibble = code & 0xF).
__device__ __forceinline__ uint32_t pack8_magic(const float (&m)[8]) {
  uint32_t b[4];
#pragma unroll
  for (int k = 0; k < 4; k++)
    b[k] = (__float_as_uint(m[2 * k]) & 0xFu) | ((__float_as_uint(m[2 * k + 1]) & 0xFu) << 4);
  return prmt(prmt(b[0], b[1], 0x0040u), prmt(b[2], b[3], 0x0040u), 0x5410u);
}

// Quantise this lane's 64 rotated values of a row; q[2j], q[2j+1] = packed codes of
// chunk j.  Returns the fp16 scale bits (identical on both lanes of the row).
//
// Codes are round-half-even of y / s with s the stored fp16 scale.  Fast path (a normal,
// unsaturated s, so |y/s| <= 7.004): multiply the unscaled butterfly output z by
// fl(c_b * fl(1/s)) and round with the magic addend; the product is within 2^-19 of y/s,
// so the result is exact unless the fraction is within 2^-19 of one half.  A group of 8 values with such a near-tie -- frequent for rows that are
// not rotated, whose fp16 values meet exact ties -- and every group when s is subnormal
// or saturated is recomputed exactly without dividing: k = floor(y*r) is within one of
// the true floor, and (k + 1/2)*s is exact in fp32 (an fp16 scale times a number of 5
// bits), so comparing y with it chooses between k and k + 1, an exact tie going to the
// even one.  (If y*r fell on the wrong side of an integer n, y/s is within 2^-16 of n
// and both candidates' half points place it at n.)  Codes are clamped to [-8, 7].
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint16_t quantise(const float (&z)[64], float cb, unsigned pmask,
                                             uint32_t (&q)[8]) {
  // m = max |y| = fl(c_b * max |z|): rounding is monotonic, so scaling after the max gives
  // the max of the scaled values.
  float zmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 64; i += 2) zmax = max3(zmax, fabsf(z[i]), fabsf(z[i + 1]));
  zmax = fmaxf(zmax, __shfl_xor_sync(pmask, zmax, 1));
  const float m = __fmul_rn(cb, zmax);
  const float s32 = __fdiv_rn(m, 7.0f);
  const bool sat = s32 > 65504.0f;
  const __half sh = sat ? __ushort_as_half(0x7BFF) : __float2half_rn(s32);
  const float s = __half2float(sh);
  if (s == 0.0f) {  // an all-zero row (or a scale that underflows): every code is 0
#pragma unroll
    for (int w = 0; w < 8; w++) q[w] = 0u;
    return __half_as_ushort(sh);
  }
  const bool normal = !sat && s >= 6.103515625e-05f;
  const float r = __frcp_rn(s);
  // Fast path on z directly: t = z * fl(c_b * r) is within 4 roundings (< 2^-19 for
  // |y/s| <= 7.004) of y / s.
  const float rz = __fmul_rn(cb, r);
  const float hs = 0.5f * s;
#pragma unroll
  for (int c8 = 0; c8 < 8; c8++) {
    float mg[8];
    float dmax = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float t0 = z[8 * c8 + e], t1 = z[8 * c8 + e + 1];
      mul2(t0, t1, rz);
      float m0 = t0, m1 = t1;
      fma2(m0, m1, 1.0f, kMagic, kMagic);           // t + 1.5*2^23, rounded: rint
      float r0 = m0, r1 = m1;
      fma2(r0, r1, 1.0f, -kMagic, -kMagic);         // the integer, exactly
      float d0 = r0, d1 = r1;
      fma2(d0, d1, -1.0f, t0, t1);                  // t - rint(t), exactly
      dmax = max3(dmax, fabsf(d0), fabsf(d1));
      mg[e] = m0;
      mg[e + 1] = m1;
    }
    if (!normal || !(dmax < 0.5f - 0x1p-19f)) {
#pragma unroll
      for (int e = 0; e < 8; e++) {
        const float y = __fmul_rn(z[8 * c8 + e], cb);  // the rotated value
        const float k = floorf(__fmul_rn(y, r));
        const float h = __fmaf_rn(k, s, hs);  // (k + 1/2) * s, exact
        const bool odd = (__float_as_uint(__fadd_rn(k, kMagic)) & 1u) != 0u;
        const bool up = y > h || (y == h && odd);
        const float t = fminf(fmaxf(up ? k + 1.0f : k, -8.0f), 7.0f);
        mg[e] = __fadd_rn(t, kMagic);
      }
    }
    q[c8] = pack8_magic(mg);
  }
  return __half_as_ushort(sh);
}

// The K or V row r of the call: (token, head) pair r / 2, tensor r % 2.
__device__ __forceinline__ const __half* row_src(const AppendParams& p, long long r) {
  return ((r & 1) ? p.v : p.k) + static_cast<size_t>(r >> 1) * kD;
}

// Persistent: CTA i takes row blocks i, i + grid, ...; the loads of a lane's next row are
// issued before the current row is rotated, quantised and stored, so they are in flight
// while it computes.
template <int BLOCK>
__global__ void __launch_bounds__(kThreads, 2) append_kernel(AppendParams p) {
  // The next kernel may start its own prologue; the pool stores below wait for every
  // earlier kernel (griddep_wait), so they never race with a decode still reading.
  griddep_launch_dependents();
  const int l = threadIdx.x & 1;
  // Shuffles never leave the lane pair of a row, so they name only those two lanes.
  const unsigned pmask = 0x3u << (threadIdx.x & 30);
  const long long nrows = 2LL * p.total_new_tokens * p.num_kv_heads;
  const long long nblk = (nrows + kRowsPerBlock - 1) / kRowsPerBlock;
  const int r_in = threadIdx.x >> 1;
  long long rb = blockIdx.x;
  u32x8 raw[4];
  {
    const long long row = rb * kRowsPerBlock + r_in;
    if (row < nrows) load_row(row_src(p, row), l, raw);
  }
  bool waited = false;
  for (; rb < nblk; rb += gridDim.x) {
    const long long row = rb * kRowsPerBlock + r_in;
    const long long row_next = (rb + gridDim.x) * kRowsPerBlock + r_in;
    u32x8 nxt[4];
    if (rb + gridDim.x < nblk && row_next < nrows) load_row(row_src(p, row_next), l, nxt);
    if (row < nrows) {  // both lanes of a row take the same branch
      const long long pair = row >> 1;
      const int kv = static_cast<int>(row & 1);
      const int t = static_cast<int>(pair / p.num_kv_heads);
      const int h = static_cast<int>(pair % p.num_kv_heads);

      float x[64];
      rotate_row<BLOCK>(raw, l, pmask, x);

      // Sequence of token t: the b with cu[b] <= t < cu[b+1] (binary search).
      int lo = 0, hi = p.batch;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.cu_new_tokens + mid) <= t) lo = mid; else hi = mid;
      }
      const int b = lo;
      const int pos = __ldg(p.seq_lens + b) + (t - __ldg(p.cu_new_tokens + b));
      const int lp = pos / p.page_size;
      int page = -1;
      if (pos >= 0 && lp < p.max_pages_per_seq)
        page = __ldg(p.page_table + static_cast<size_t>(b) * p.max_pages_per_seq + lp);
      const bool ok = pos >= 0 && lp < p.max_pages_per_seq && page >= 0 && page < p.num_pages;

      uint32_t q[8];
      const uint16_t sbits = quantise(x, p.cb, pmask, q);
      if (!waited) {
        griddep_wait();
        waited = true;
      }
      if (!ok) {
        if (l == 0 && kv == 0)
          atomicOr(p.status, (pos < 0 || lp >= p.max_pages_per_seq) ? KVQ_DEV_BAD_POS_BIT
                                                                      : KVQ_DEV_BAD_PAGE_BIT);
      } else {
        const int S = p.page_size;
        const int slot = pos - lp * S;
        uint8_t* blk = p.pool_layer + (static_cast<size_t>(page) * p.num_kv_heads + h) *
                                          (static_cast<size_t>(S) * (kD + 4));
        uint8_t* crow =
            blk + static_cast<size_t>(kv) * S * (kD / 2) + static_cast<size_t>(slot) * (kD / 2);
#pragma unroll
        for (int j = 0; j < 4; j++)
          *reinterpret_cast<uint2*>(crow + 8 * (2 * j + l)) = make_uint2(q[2 * j], q[2 * j + 1]);
        if (l == 0)
          *reinterpret_cast<uint16_t*>(blk + static_cast<size_t>(S) * kD +
                                       static_cast<size_t>(kv) * S * 2 + static_cast<size_t>(slot) * 2) =
              sbits;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; j++) raw[j] = nxt[j];
  }
}

}  // namespace

int launch_append(const AppendParams& p, int block, int num_sms, cudaStream_t stream) {
  const long long nrows = 2LL * p.total_new_tokens * p.num_kv_heads;
  if (nrows == 0) return 0;
  const long long nblk = (nrows + kRowsPerBlock - 1) / kRowsPerBlock;
  if (nblk > 0x7fffffffLL) return -1;
  // One wave of persistent CTAs (2 per SM), or fewer for a small call.
  const long long grid = nblk < 2LL * num_sms ? nblk : 2LL * num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  switch (block) {
    case 1: e = cudaLaunchKernelEx(&cfg, append_kernel<1>, p); break;
    case 32: e = cudaLaunchKernelEx(&cfg, append_kernel<32>, p); break;
    case 64: e = cudaLaunchKernelEx(&cfg, append_kernel<64>, p); break;
    case 128: e = cudaLaunchKernelEx(&cfg, append_kernel<128>, p); break;
    default: return -1;
  }
  return e == cudaSuccess ? 0 : -2;
}

}  // namespace kvq

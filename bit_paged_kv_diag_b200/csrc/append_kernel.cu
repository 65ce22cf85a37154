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
// Work decomposition.  One group of 4 lanes handles one (token, KV head) pair: both
// its K row and its V row (128 fp16 channels each).  Lane l of the group holds
// channels [16l, 16l+16) and [64+16l, 64+16l+16), loaded as two 256-bit reads, so the
// 4 lanes read the row's 256 bytes as two fully used 128-byte lines.  In channel-index
// bits, bits 0-3 and bit 6 are inside a lane and bits 4-5 are across lanes, so the
// butterfly stages h = 1, 2, 4, 8 and 64 are register-only and stages h = 16, 32 are
// warp shuffles (xor 1, xor 2).  The stage order and every add/subtract are those of
// the fixed-order fp32 butterfly (stages h = 1, 2, ..., b/2, pairs (i, i+h) with bit h
// of i clear -> (a+c, a-c)), then one multiply by the fp32 constant nearest 1/sqrt(b),
// each as a single IEEE operation, so rotated values, scales and codes are bit-exact
// with any implementation of the same fixed-order butterfly.
//
// The row's absmax is a 2-step shuffle reduction over the group; the scale is
// fp16_rn(max/7) (IEEE division); codes are round-half-even of y / s (IEEE division by
// the stored fp16 scale), clamped to [-8, 7], packed two per byte (low nibble = even
// channel).  After one 8-byte exchange with the neighbouring lane, every lane holds 16
// contiguous code bytes and writes them with one 128-bit store; lanes 0 and 1 store the
// K and V scales.
#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kD = 128;
constexpr int kPairsPerBlock = 64;            // (token, head) pairs per CTA
constexpr int kThreads = kPairsPerBlock * 4;  // 4 lanes per pair

// x[0..15] = channels [16l, 16l+16), x[16..31] = channels [64+16l, 64+16l+16).
template <int BLOCK>
__device__ __forceinline__ void rotate_row(float (&x)[32], int lane4, unsigned gmask, float cb) {
  // In-lane stages: h = 1, 2, 4, 8 act on bits 0-3 of the in-group index.
#pragma unroll
  for (int h = 1; h <= 8; h *= 2) {
    if (h < BLOCK) {
#pragma unroll
      for (int grp = 0; grp < 2; grp++) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
          if (i & h) continue;
          const float a = x[grp * 16 + i];
          const float c = x[grp * 16 + i + h];
          x[grp * 16 + i] = __fadd_rn(a, c);
          x[grp * 16 + i + h] = __fsub_rn(a, c);
        }
      }
    }
  }
  // Cross-lane stages h = 16 (partner lane ^ 1) and h = 32 (partner lane ^ 2).  The
  // lane holding the lower index computes own + other; the upper one other - own.  A
  // single fused multiply-add with a +-1 multiplier rounds once, so
  // fma(own, -1, other) is bit-identical to the IEEE difference other - own.
#pragma unroll
  for (int s = 0; s < 2; s++) {
    const int h = 16 << s;
    if (h < BLOCK) {
      const int bit = 1 << s;
      const float sgn = (lane4 & bit) ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < 32; i++) {
        const float other = __shfl_xor_sync(gmask, x[i], bit);
        x[i] = __fmaf_rn(x[i], sgn, other);
      }
    }
  }
  // In-lane stage h = 64: channel 16l+i pairs with channel 64+16l+i.
  if (64 < BLOCK) {
#pragma unroll
    for (int i = 0; i < 16; i++) {
      const float a = x[i];
      const float c = x[16 + i];
      x[i] = __fadd_rn(a, c);
      x[16 + i] = __fsub_rn(a, c);
    }
  }
#pragma unroll
  for (int i = 0; i < 32; i++) x[i] = __fmul_rn(x[i], cb);
}

__device__ __forceinline__ void load_row(const __half* row, int lane4, float (&x)[32]) {
#pragma unroll
  for (int j = 0; j < 2; j++) {
    // 32 bytes = 16 channels starting at channel 64j + 16*lane4.
    const u32x8 r = ldg_256_stream(row + 64 * j + 16 * lane4);
#pragma unroll
    for (int w = 0; w < 8; w++) {
      const __half2 h2 = *reinterpret_cast<const __half2*>(&r.w[w]);
      const float2 f = __half22float2(h2);
      x[16 * j + 2 * w] = f.x;
      x[16 * j + 2 * w + 1] = f.y;
    }
  }
}

// Quantise the rotated row; returns the fp16 scale bits and the packed codes, 8
// channels per word: q[0], q[1] = group A (channels 16l..16l+15), q[2], q[3] = group
// B (channels 64+16l..64+16l+15).
__device__ __forceinline__ uint16_t quantise_row(const float (&y)[32], unsigned gmask,
                                                 uint32_t (&q)[4]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; i++) m = fmaxf(m, fabsf(y[i]));
  m = fmaxf(m, __shfl_xor_sync(gmask, m, 1));
  m = fmaxf(m, __shfl_xor_sync(gmask, m, 2));
  const float s32 = __fdiv_rn(m, 7.0f);
  const __half sh = (s32 > 65504.0f) ? __ushort_as_half(0x7BFF) : __float2half_rn(s32);
  const float s = __half2float(sh);
#pragma unroll
  for (int w = 0; w < 4; w++) q[w] = 0u;
  if (s != 0.0f) {
#pragma unroll
    for (int i = 0; i < 32; i++) {
      float t = rintf(__fdiv_rn(y[i], s));
      t = fminf(fmaxf(t, -8.0f), 7.0f);
      const uint32_t nib = static_cast<uint32_t>(static_cast<int>(t)) & 0xFu;
      q[i / 8] |= nib << (4 * (i % 8));
    }
  }
  return __half_as_ushort(sh);
}

template <int BLOCK>
__global__ void __launch_bounds__(kThreads) append_kernel(AppendParams p) {
  const int lane4 = threadIdx.x & 3;
  // Shuffles never leave the 4-lane group, so they name only the group's lanes.
  const unsigned gmask = 0xFu << (threadIdx.x & 28);
  const long long pair = static_cast<long long>(blockIdx.x) * kPairsPerBlock + (threadIdx.x >> 2);
  const long long npairs = static_cast<long long>(p.total_new_tokens) * p.num_kv_heads;
  // Whole groups of 4 share validity and shuffle only among themselves, so a group
  // past the end may leave early.
  if (pair >= npairs) return;
  const int t = static_cast<int>(pair / p.num_kv_heads);
  const int h = static_cast<int>(pair % p.num_kv_heads);

  // Issue the K/V loads first; the page lookup below overlaps their latency.
  float xk[32], xv[32];
  const size_t row_off = (static_cast<size_t>(t) * p.num_kv_heads + h) * kD;
  load_row(p.k + row_off, lane4, xk);
  load_row(p.v + row_off, lane4, xv);

  // Sequence of token t: the b with cu[b] <= t < cu[b+1] (binary search).
  int lo = 0, hi = p.batch;  // invariant: cu[lo] <= t < cu[hi]
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

  rotate_row<BLOCK>(xk, lane4, gmask, p.cb);
  rotate_row<BLOCK>(xv, lane4, gmask, p.cb);
  uint32_t qk[4], qv[4];
  const uint16_t sk = quantise_row(xk, gmask, qk);
  const uint16_t sv = quantise_row(xv, gmask, qv);

  if (!ok) {
    if (lane4 == 0)
      atomicOr(p.status, (pos < 0 || lp >= p.max_pages_per_seq) ? KVQ_DEV_BAD_POS_BIT
                                                                  : KVQ_DEV_BAD_PAGE_BIT);
    return;
  }
  const int S = p.page_size;
  const int slot = pos - lp * S;
  uint8_t* blk = p.pool_layer + (static_cast<size_t>(page) * p.num_kv_heads + h) *
                                    (static_cast<size_t>(S) * (kD + 4));
  // Exchange 8 bytes with the neighbour so each lane owns 16 contiguous code bytes:
  // even lane l stores bytes [8l, 8l+16) = (own A, neighbour A); odd lane l stores
  // bytes [24+8l, 40+8l) = (neighbour B, own B).
  const bool odd = lane4 & 1;
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    const uint32_t* q = kv == 0 ? qk : qv;
    const uint32_t s0 = odd ? q[0] : q[2], s1 = odd ? q[1] : q[3];
    const uint32_t r0 = __shfl_xor_sync(gmask, s0, 1);
    const uint32_t r1 = __shfl_xor_sync(gmask, s1, 1);
    uint8_t* row = blk + static_cast<size_t>(kv) * S * (kD / 2) + static_cast<size_t>(slot) * (kD / 2);
    if (!odd) stg_128(row + 8 * lane4, q[0], q[1], r0, r1);
    else stg_128(row + 24 + 8 * lane4, r0, r1, q[2], q[3]);
  }
  if (lane4 < 2) {
    uint8_t* sp = blk + static_cast<size_t>(S) * kD + static_cast<size_t>(lane4) * S * 2 +
                  static_cast<size_t>(slot) * 2;
    *reinterpret_cast<uint16_t*>(sp) = lane4 == 0 ? sk : sv;
  }
}

}  // namespace

int launch_append(const AppendParams& p, int block, cudaStream_t stream) {
  const long long npairs = static_cast<long long>(p.total_new_tokens) * p.num_kv_heads;
  if (npairs == 0) return 0;
  const long long grid = (npairs + kPairsPerBlock - 1) / kPairsPerBlock;
  if (grid > 0x7fffffffLL) return -1;
  switch (block) {
    case 32: append_kernel<32><<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(p); break;
    case 64: append_kernel<64><<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(p); break;
    case 128: append_kernel<128><<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(p); break;
    default: return -1;
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

}  // namespace kvq

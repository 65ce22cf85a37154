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
// KV head) "unit", numbered unit-major.  CTA k of C takes the contiguous tile range
// [k*T/C, (k+1)*T/C) of the T tiles, so every CTA streams the same number of bytes
// whatever the length mix.  Its 4 warps take the range's tiles of each unit in turn
// (tile xs + w, xs + w + 4, ...), each keeping an online-softmax state; at the end of
// each unit the warps merge through shared memory.  A unit inside one CTA is finished
// there (normalise, inverse rotation, fp16 store).  A unit spanning several CTAs leaves
// one (o', m, l) partial per CTA in scratch slot unit + k (unique along the staircase of
// ranges); the last CTA to arrive (an atomic counter per unit, reset after use) merges
// them and finishes the unit.
//
// Loads.  Each warp owns a ring of 3 shared-memory slots of one tile each.  Per tile one
// lane per page issues a 1-D bulk copy (cp.async.bulk, TMA engine, no multicast) of the
// contiguous (page, head) block -- codes and scales together -- into a slot, completing
// on the slot's mbarrier; page ids three tiles ahead are read while the current tile
// computes.
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
// the two parts sit in neighbouring columns, for G = 8 two MMAs accumulate them.  The GQA group is the N = 8
// side of both products; the dequantised cache is the M side.  The K scale multiplies the
// fp32 score of its token; softmax runs in the log2 domain with exp2.
#include <cuda_fp16.h>
#include <math_constants.h>
#include <stdint.h>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kD = 128;
constexpr int kSlotBytes = kTileTokens * (kD + 4);  // 4224: one tile of codes + scales
constexpr int kWarps = 4;                           // warps per CTA
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

// One (sequence, KV head) unit and its place in the tile sequence.
struct Unit {
  int b, h;       // sequence, KV head
  int n;          // tiles in the unit
  int L;          // tokens (clamped to the page budget)
  long long U;    // global index of the unit's first tile
};

__device__ __forceinline__ void unit_of_tile(Unit& u, long long x, const int32_t* pre,
                                             const DecodeParams& p) {
  int lo = 0, hi = p.batch;  // pre[lo]*Hkv <= x < pre[hi]*Hkv
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<long long>(pre[mid]) * p.num_kv_heads <= x) lo = mid; else hi = mid;
  }
  u.b = lo;
  u.n = pre[lo + 1] - pre[lo];
  const long long base = static_cast<long long>(pre[lo]) * p.num_kv_heads;
  u.h = static_cast<int>((x - base) / u.n);
  u.U = base + static_cast<long long>(u.h) * u.n;
  u.L = clamp_len(__ldg(p.seq_lens + u.b), p.max_pages_per_seq * p.page_size, p.status);
}

// The next non-empty unit.  Callers only ask while one exists.
__device__ __forceinline__ void unit_next(Unit& u, const int32_t* pre, const DecodeParams& p) {
  if (++u.h == p.num_kv_heads) {
    u.h = 0;
    do { ++u.b; } while (u.b < p.batch && pre[u.b + 1] == pre[u.b]);
    if (u.b >= p.batch) return;
    u.n = pre[u.b + 1] - pre[u.b];
    u.L = clamp_len(__ldg(p.seq_lens + u.b), p.max_pages_per_seq * p.page_size, p.status);
  }
  u.U = static_cast<long long>(pre[u.b]) * p.num_kv_heads + static_cast<long long>(u.h) * u.n;
}

// CTA whose tile range holds tile x (ranges [k*T/C, (k+1)*T/C)).
__device__ __forceinline__ long long cta_of(long long x, long long T, long long C) {
  return ((x + 1) * C - 1) / T;
}

// A warp's walk over its tiles: units overlapping [X0, X1), tiles xs + w + 4i of each.
struct Walk {
  Unit u;
  long long x, xe;
  bool valid;
};

__device__ __forceinline__ void walk_settle(Walk& wk, long long X1, int w, const int32_t* pre,
                                            const DecodeParams& p) {
  while (wk.x >= wk.xe) {
    if (wk.xe >= X1) {
      wk.valid = false;
      return;
    }
    unit_next(wk.u, pre, p);
    wk.x = wk.u.U + w;
    wk.xe = min(X1, wk.u.U + wk.u.n);
  }
}

// ------------------------------------------------------------------- copies --
// Page id lane `lane` needs for tile k of unit u (or -1): for pages of <= 32 tokens the
// tile's pages (<= 2), else the page holding the tile.
template <int SEFF>
__device__ __forceinline__ int tile_page_id(const Unit& u, long long k, int lane,
                                            const DecodeParams& p) {
  const int S = p.page_size;
  const int t0 = static_cast<int>(k) * kTileTokens;
  int npg = 1;
  if (S <= kTileTokens) npg = (min(t0 + kTileTokens, u.L) - 1) / S - t0 / S + 1;
  if (lane >= npg) return -1;
  return __ldg(p.page_table + static_cast<size_t>(u.b) * p.max_pages_per_seq + t0 / S + lane);
}

// Issue the bulk copies of tile k of unit u into a ring slot (the whole warp calls).
// The slot holds a virtual page of SEFF = min(S, 32) token slots per copied page,
// [K codes][V codes][K scales][V scales], the pool's own block layout.
template <int SEFF>
__device__ __forceinline__ void tile_issue(const Unit& u, long long k, int pid, uint32_t slot,
                                           uint32_t bar, int lane, uint64_t pol,
                                           const DecodeParams& p) {
  const int S = p.page_size;
  const uint32_t blk_bytes = static_cast<uint32_t>(S) * (kD + 4);
  const int t0 = static_cast<int>(k) * kTileTokens;
  int npg = 1;
  uint32_t total = kSlotBytes;
  if (S <= kTileTokens) {
    npg = (min(t0 + kTileTokens, u.L) - 1) / S - t0 / S + 1;
    total = npg * blk_bytes;
  }
  const bool bad = lane < npg && (pid < 0 || pid >= p.num_pages);
  if (__any_sync(kFull, bad) && lane == 0) atomicOr(p.status, KVQ_DEV_BAD_PAGE_BIT);
  if (bad) pid = 0;  // keep the barrier's byte count; the status word flags the result
  if (lane == 0) mbar_arrive_expect_tx(bar, total);
  __syncwarp();
  if (S <= kTileTokens) {
    if (lane < npg)
      bulk_copy_g2s(slot + lane * blk_bytes,
                    p.pool_layer + (static_cast<size_t>(pid) * p.num_kv_heads + u.h) * blk_bytes,
                    blk_bytes, bar, pol);
  } else {
    const int pid0 = __shfl_sync(kFull, pid, 0);
    const size_t o = static_cast<size_t>(t0 % S);  // first token of the tile in the page
    const uint8_t* blk = p.pool_layer + (static_cast<size_t>(pid0) * p.num_kv_heads + u.h) * blk_bytes;
    if (lane == 0) bulk_copy_g2s(slot, blk + o * 64, 2048, bar, pol);
    if (lane == 1) bulk_copy_g2s(slot + 2048, blk + static_cast<size_t>(S) * 64 + o * 64, 2048, bar, pol);
    if (lane == 2) bulk_copy_g2s(slot + 4096, blk + static_cast<size_t>(S) * 128 + o * 2, 64, bar, pol);
    if (lane == 3) bulk_copy_g2s(slot + 4160, blk + static_cast<size_t>(S) * 130 + o * 2, 64, bar, pol);
  }
}

// ------------------------------------------------------------------------ q --
template <int G>
struct QFrag {
  static constexpr int NQ = (G == 8) ? 2 : 1;  // queries owned by one thread
  // int8 B fragments per k32 chunk jj: [jj][0] = k 4c..4c+3, [jj][1] = k 16+4c..16+4c+3.
  // G <= 4: A = column g holds slice 1 (g even) or 2 (g odd) of query g/2, B = slice 3
  // (g even) or zero.  G == 8: A, B, C = slices 1, 2, 3 of query g.
  uint32_t A[4][2], B[4][2], C[4][2];
  float sf[NQ];  // M / 1024 of the owned queries
};

// Raw fp16 q row of this thread's column: channels [32c, 32c+32).
template <int G>
__device__ __forceinline__ void load_q_raw(uint4 (&raw)[4], const Unit& u, int lane,
                                           const DecodeParams& p) {
  const int g = lane >> 2, c = lane & 3;
  const int qi = (G == 8) ? g : (g >> 1);
  if (qi < G) {
    const uint4* src = reinterpret_cast<const uint4*>(
        p.q + (static_cast<size_t>(u.b) * p.num_kv_heads * G + u.h * G + qi) * kD + 32 * c);
#pragma unroll
    for (int v = 0; v < 4; v++) raw[v] = __ldg(src + v);
  } else {
#pragma unroll
    for (int v = 0; v < 4; v++) raw[v] = make_uint4(0u, 0u, 0u, 0u);
  }
}

__device__ __forceinline__ uint32_t int8x4(const float (&m)[32], int i0, int step) {
  // Low bytes of four magic-rounded sums (each holds an integer in [-64, 64]).
  const uint32_t b0 = __float_as_uint(m[i0]), b1 = __float_as_uint(m[i0 + step]);
  const uint32_t b2 = __float_as_uint(m[i0 + 2 * step]), b3 = __float_as_uint(m[i0 + 3 * step]);
  return prmt(prmt(b0, b1, 0x0040u), prmt(b2, b3, 0x0040u), 0x5410u);
}

// Rotate q (same fixed-order butterfly: bits 0-4 in registers, bits 5-6 across the 4
// lanes of the row group), scale by c_b * softmax_scale * log2(e), cut into int8 slices.
template <int G>
__device__ __forceinline__ void make_qfrag(QFrag<G>& f, const uint4 (&raw)[4], int lane,
                                           const DecodeParams& p) {
  const int g = lane >> 2, c = lane & 3;
  float x[32];
#pragma unroll
  for (int v = 0; v < 4; v++) {
    const uint32_t w[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
      x[8 * v + 2 * e] = t.x;
      x[8 * v + 2 * e + 1] = t.y;
    }
  }
  const int block = p.hadamard_block;
#pragma unroll
  for (int h = 1; h <= 16; h *= 2) {
    if (h < block) {
#pragma unroll
      for (int i = 0; i < 32; i++) {
        if (i & h) continue;
        const float a = x[i], d = x[i + h];
        x[i] = __fadd_rn(a, d);
        x[i + h] = __fsub_rn(a, d);
      }
    }
  }
#pragma unroll
  for (int s = 0; s < 2; s++) {
    if ((32 << s) < block) {
      const int bit = 1 << s;
      const float sgn = (c & bit) ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < 32; i++) {
        const float other = __shfl_xor_sync(kFull, x[i], bit);
        x[i] = __fmaf_rn(x[i], sgn, other);
      }
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; i++) {
    x[i] = __fmul_rn(__fmul_rn(x[i], p.cb), p.q_scale);
    amax = fmaxf(amax, fabsf(x[i]));
  }
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
  // M = the smallest power of two >= amax (1 for a zero row).
  float M = 1.0f;
  if (amax > 1e-30f) {
    const uint32_t bits = __float_as_uint(amax);
    M = (bits & 0x7FFFFFu) ? __uint_as_float((bits & 0x7F800000u) + 0x00800000u) : amax;
  }
  const float inv = __fdiv_rn(64.0f, M);  // exact: powers of two
  float m1[32], m2[32], m3[32];
#pragma unroll
  for (int i = 0; i < 32; i++) {
    const float t = x[i] * inv;                 // |t| <= 64, exact scaling
    m1[i] = t + kMagic;                         // rint(t) in the low mantissa bits
    const float r1 = (t - (m1[i] - kMagic)) * 128.0f;  // |r1| <= 64, exact
    m2[i] = r1 + kMagic;
    const float r2 = (r1 - (m2[i] - kMagic)) * 128.0f;
    m3[i] = r2 + kMagic;
  }
  uint32_t s1[4][2], s2[4][2], s3[4][2];
#pragma unroll
  for (int jj = 0; jj < 4; jj++) {
    // k = 4c + e <-> channel 32c + 8jj + 2e; k = 16 + 4c + e <-> channel 32c + 8jj + 2e + 1.
    s1[jj][0] = int8x4(m1, 8 * jj, 2);
    s1[jj][1] = int8x4(m1, 8 * jj + 1, 2);
    s2[jj][0] = int8x4(m2, 8 * jj, 2);
    s2[jj][1] = int8x4(m2, 8 * jj + 1, 2);
    s3[jj][0] = int8x4(m3, 8 * jj, 2);
    s3[jj][1] = int8x4(m3, 8 * jj + 1, 2);
  }
  const float sf_col = M * (1.0f / 1024.0f);
#pragma unroll
  for (int jj = 0; jj < 4; jj++)
#pragma unroll
    for (int e = 0; e < 2; e++) {
      if (G == 8) {
        f.A[jj][e] = s1[jj][e];
        f.B[jj][e] = s2[jj][e];
        f.C[jj][e] = s3[jj][e];
      } else {
        const bool col_ok = (g >> 1) < G;
        f.A[jj][e] = col_ok ? ((g & 1) ? s2[jj][e] : s1[jj][e]) : 0u;
        f.B[jj][e] = (col_ok && !(g & 1)) ? s3[jj][e] : 0u;
        f.C[jj][e] = 0u;
      }
    }
  if (G == 8) {
    f.sf[0] = __shfl_sync(kFull, sf_col, 4 * (2 * c));
    f.sf[QFrag<G>::NQ - 1] = __shfl_sync(kFull, sf_col, 4 * (2 * c + 1));
  } else {
    f.sf[0] = __shfl_sync(kFull, sf_col, 8 * c);
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

__device__ __forceinline__ float half_at(uint32_t addr) {
  return __half2float(__ushort_as_half(lds_u16(addr)));
}

// One tile (2 k-steps of 16 tokens) from a ring slot; ntok valid tokens.
template <int G, int SEFF>
__device__ __forceinline__ void tile_compute(State<G>& st, const QFrag<G>& qf, uint32_t slot,
                                             int ntok, int lane) {
  constexpr int NQ = State<G>::NQ;
  const int g = lane >> 2, c = lane & 3;
  const int tau0 = (g < 4) ? g : g + 4;  // token of A row g (QK^T)
  const int tau1 = tau0 + 4;             // token of A row g + 8
  float sc[2][NQ][2];                    // scores (log2 domain): [k-step][query][row]

#pragma unroll
  for (int j = 0; j < 2; j++) {
    const uint32_t pbase = slot + (16 * j / SEFF) * (SEFF * 132);
    const int sl = (16 * j) % SEFF;
    const uint32_t kb = pbase + sl * 64;
    const uint4 ka = lds_128(kb + tau0 * 64 + 16 * c);
    const uint4 kc = lds_128(kb + tau1 * 64 + 16 * c);
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
    const uint32_t skb = pbase + SEFF * 128 + sl * 2;
    const float sk0 = half_at(skb + tau0 * 2), sk1 = half_at(skb + tau1 * 2);
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
          sc[j][qq][r] = (r ? v1 : v0) ? v * (r ? sk1 : sk0) * qf.sf[qq] : -CUDART_INF_F;
        }
    } else {
      // Column 2c = slices 1 (A) and 3 (B) of query c, 2c+1 = slice 2 (A) of query c.
      const float va = static_cast<float>(accA[0]) + static_cast<float>(accA[1] * 128 + accB[0]) * k14;
      const float vc = static_cast<float>(accA[2]) + static_cast<float>(accA[3] * 128 + accB[2]) * k14;
      sc[j][0][0] = v0 ? va * sk0 * qf.sf[0] : -CUDART_INF_F;
      sc[j][0][1] = v1 ? vc * sk1 * qf.sf[0] : -CUDART_INF_F;
    }
  }

  // Online softmax over the tile (log2 domain).
  float alpha[NQ];
  bool rescale = false;
#pragma unroll
  for (int qq = 0; qq < NQ; qq++) {
    float mx = fmaxf(fmaxf(sc[0][qq][0], sc[0][qq][1]), fmaxf(sc[1][qq][0], sc[1][qq][1]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
    const float mnew = fmaxf(st.m[qq], mx);
    alpha[qq] = exp2f(st.m[qq] - mnew);
    rescale |= alpha[qq] != 1.0f;
    st.m[qq] = mnew;
    float ps = 0.0f;
#pragma unroll
    for (int j = 0; j < 2; j++)
#pragma unroll
      for (int r = 0; r < 2; r++) {
        sc[j][qq][r] = exp2f(sc[j][qq][r] - mnew);
        ps += sc[j][qq][r];
      }
    st.l[qq] = st.l[qq] * alpha[qq] + ps;
  }
  if (__any_sync(kFull, rescale)) {
#pragma unroll
    for (int i = 0; i < 8; i++) {
      // G <= 4: columns 2c, 2c+1 are query c's hi and lo parts; G == 8: queries 2c, 2c+1.
      st.o[i][0] *= alpha[0];
      st.o[i][2] *= alpha[0];
      st.o[i][1] *= alpha[NQ - 1];
      st.o[i][3] *= alpha[NQ - 1];
    }
  }

  // PV.  B fragment of thread (g, c): tokens c, c+4 (b0) and c+8, c+12 (b1) of the
  // k-step for column g, taken from the lanes that scored them (rows c and c + 4 of
  // the QK^T fragment).
  const int srcA = 4 * c + (g >> 1);
  const int srcB = srcA + 16;
#pragma unroll
  for (int j = 0; j < 2; j++) {
    const uint32_t pbase = slot + (16 * j / SEFF) * (SEFF * 132);
    const int sl = (16 * j) % SEFF;
    const uint32_t vb = pbase + SEFF * 64 + sl * 64;
    const uint32_t svb = pbase + SEFF * 130 + sl * 2;
    const float sv0 = half_at(svb + tau0 * 2), sv1 = half_at(svb + tau1 * 2);
    const bool v0 = 16 * j + tau0 < ntok, v1 = 16 * j + tau1 < ntok;
    // P' = p * s_v carried as fp16 hi + lo (relative precision ~2^-22).
    uint32_t bh0, bh1, bl0 = 0u, bl1 = 0u;
    if (G == 8) {
      uint32_t xh[2], xl[2];
#pragma unroll
      for (int qq = 0; qq < 2; qq++) {
        const float p0 = v0 ? sc[j][qq][0] * sv0 : 0.0f, p1 = v1 ? sc[j][qq][1] * sv1 : 0.0f;
        const __half h0 = __float2half_rn(p0), h1 = __float2half_rn(p1);
        xh[qq] = pack_half2(h0, h1);
        xl[qq] = pack_half2(__float2half_rn(p0 - __half2float(h0)),
                            __float2half_rn(p1 - __half2float(h1)));
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
      const float p0 = v0 ? sc[j][0][0] * sv0 : 0.0f, p1 = v1 ? sc[j][0][1] * sv1 : 0.0f;
      const __half h0 = __float2half_rn(p0), h1 = __float2half_rn(p1);
      const uint32_t xh = pack_half2(h0, h1);
      const uint32_t xl = pack_half2(__float2half_rn(p0 - __half2float(h0)),
                                     __float2half_rn(p1 - __half2float(h1)));
      // Column g = 2q + part holds query q's hi (part 0) or lo (part 1) part.
      const uint32_t aH = __shfl_sync(kFull, xh, srcA), aL = __shfl_sync(kFull, xl, srcA);
      const uint32_t cH = __shfl_sync(kFull, xh, srcB), cL = __shfl_sync(kFull, xl, srcB);
      bh0 = (g & 1) ? aL : aH;
      bh1 = (g & 1) ? cL : cH;
      if ((g >> 1) >= G) bh0 = bh1 = 0u;
    }
    // V rows of tokens c, c+4, c+8, c+12; this thread's channels [16g, 16g+16).
    const uint2 t0 = lds_64(vb + (c + 0) * 64 + 8 * g);
    const uint2 t1 = lds_64(vb + (c + 4) * 64 + 8 * g);
    const uint2 t2 = lds_64(vb + (c + 8) * 64 + 8 * g);
    const uint2 t3 = lds_64(vb + (c + 12) * 64 + 8 * g);
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

// Warp partial (owned queries) -> shared merge buffer buf[w][qi][kPartStride].
template <int G>
__device__ __forceinline__ void state_to_smem(const State<G>& st, float* buf, int w, int lane) {
  constexpr int NQ = State<G>::NQ;
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int qq = 0; qq < NQ; qq++) {
    float l = st.l[qq];
    l += __shfl_xor_sync(kFull, l, 4);
    l += __shfl_xor_sync(kFull, l, 8);
    l += __shfl_xor_sync(kFull, l, 16);
    const int qi = (G == 8) ? 2 * c + qq : c;
    if (qi >= G) continue;
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
    float* rec = buf + (w * G + qi) * kPartStride;
    float4* dst = reinterpret_cast<float4*>(rec + 16 * g);
#pragma unroll
    for (int e = 0; e < 4; e++) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    if (g == 0) {
      rec[kD] = st.m[qq];
      rec[kD + 1] = l;
    }
  }
}

// o'/l of one query (lane: channels 4*lane..4*lane+3) -> inverse block-diagonal
// Hadamard -> fp16 store.
__device__ __forceinline__ void finish_query(const float (&o)[4], float l, __half* dst, int lane,
                                             const DecodeParams& p) {
  float x[4];
#pragma unroll
  for (int e = 0; e < 4; e++) x[e] = __fdiv_rn(o[e], l);
  const int block = p.hadamard_block;
  float a, c;
  a = x[0]; c = x[1]; x[0] = a + c; x[1] = a - c;
  a = x[2]; c = x[3]; x[2] = a + c; x[3] = a - c;
  a = x[0]; c = x[2]; x[0] = a + c; x[2] = a - c;
  a = x[1]; c = x[3]; x[1] = a + c; x[3] = a - c;
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

template <int G, int SEFF>
__global__ void __launch_bounds__(kThreads, 3) decode_kernel(DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  // Bulk copies need 16-byte aligned destinations; align the ring to 128 bytes (the
  // allocation carries 128 spare bytes for this).
  uint8_t* smem = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * kSlotBytes);
  float* mbuf = reinterpret_cast<float*>(bars + kWarps * kStages);  // [kWarps][G][132]
  int32_t* pre = reinterpret_cast<int32_t*>(mbuf + kWarps * G * kPartStride);
  __shared__ int warp_sum[kWarps];
  __shared__ int running;
  __shared__ int last_flag;

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int cap = p.max_pages_per_seq * p.page_size;

  // Tiles per sequence -> exclusive prefix pre[0..batch] (block-wide scan).
  if (tid == 0) running = 0;
  __syncthreads();
  for (int base = 0; base < p.batch; base += kThreads) {
    const int i = base + tid;
    int n = 0;
    if (i < p.batch) n = (clamp_len(__ldg(p.seq_lens + i), cap, p.status) + kTileTokens - 1) / kTileTokens;
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

  // An empty sequence has no tiles: its output rows are zeros (CTAs share the writes).
  const int row_words = p.num_kv_heads * G * kD / 8;  // 16-byte words per sequence
  for (int b = blockIdx.x; b < p.batch; b += p.total_ctas)
    if (pre[b + 1] == pre[b])
      for (int i = tid; i < row_words; i += kThreads)
        reinterpret_cast<uint4*>(p.out + static_cast<size_t>(b) * p.num_kv_heads * G * kD)[i] =
            make_uint4(0u, 0u, 0u, 0u);

  const long long T = static_cast<long long>(pre[p.batch]) * p.num_kv_heads;
  const long long C = p.total_ctas;
  const long long kc = blockIdx.x;
  const long long X0 = T * kc / C, X1 = T * (kc + 1) / C;
  if (X0 >= X1) return;  // the whole CTA: nothing to do

  const uint32_t ring_s = smem_addr(ring + w * kStages * kSlotBytes);
  const uint32_t bar_s = smem_addr(bars + w * kStages);
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; s++) mbar_init(bar_s + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_policy_evict_first();

  // Producer walk: issue the first kStages tiles.
  Walk pw;
  unit_of_tile(pw.u, X0, pre, p);
  pw.x = X0 + w;
  pw.xe = min(X1, pw.u.U + pw.u.n);
  pw.valid = true;
  walk_settle(pw, X1, w, pre, p);
  int issued = 0;
  for (int s = 0; s < kStages && pw.valid; s++) {
    const int pid = tile_page_id<SEFF>(pw.u, pw.x - pw.u.U, lane, p);
    tile_issue<SEFF>(pw.u, pw.x - pw.u.U, pid, ring_s + s * kSlotBytes, bar_s + 8 * s, lane, pol, p);
    issued++;
    pw.x += kWarps;
    walk_settle(pw, X1, w, pre, p);
  }

  // Consumer: the CTA's units in order; this warp's tiles of each.
  Unit cu = pw.u;  // overwritten just below
  unit_of_tile(cu, X0, pre, p);
  long long xs = X0;
  uint4 qraw[4];
  load_q_raw<G>(qraw, cu, lane, p);
  int consumed = 0;
  bool dead = false;  // a bounded wait gave up: stop touching the ring
  State<G> st;
  QFrag<G> qf;
  while (true) {
    const long long xe = min(X1, cu.U + cu.n);
    make_qfrag<G>(qf, qraw, lane, p);
    Unit nu = cu;
    const bool has_next = xe < X1;
    if (has_next) {
      unit_next(nu, pre, p);
      load_q_raw<G>(qraw, nu, lane, p);  // prefetch the next unit's q
    }
    state_reset<G>(st);
    for (long long x = xs + w; x < xe && !dead; x += kWarps) {
      const int s = consumed % kStages;
      const uint32_t parity = static_cast<uint32_t>((consumed / kStages) & 1);
      const bool more = pw.valid;
      const int pid_next = more ? tile_page_id<SEFF>(pw.u, pw.x - pw.u.U, lane, p) : -1;
      if (!mbar_wait_bounded(bar_s + 8 * s, parity, kWaitLimitNs)) {
        dead = true;
        if (lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);
        break;
      }
      const int k = static_cast<int>(x - cu.U);
      const int ntok = min(kTileTokens, cu.L - k * kTileTokens);
      tile_compute<G, SEFF>(st, qf, ring_s + s * kSlotBytes, ntok, lane);
      consumed++;
      __syncwarp();
      if (more) {
        fence_proxy_async_smem();
        tile_issue<SEFF>(pw.u, pw.x - pw.u.U, pid_next, ring_s + s * kSlotBytes, bar_s + 8 * s,
                         lane, pol, p);
        issued++;
        pw.x += kWarps;
        walk_settle(pw, X1, w, pre, p);
      }
    }

    // Merge the 4 warps' partials of this unit.
    state_to_smem<G>(st, mbuf, w, lane);
    __syncthreads();
    const long long unit = static_cast<long long>(cu.b) * p.num_kv_heads + cu.h;
    const long long k_first = cta_of(cu.U, T, C), k_last = cta_of(cu.U + cu.n - 1, T, C);
    const bool alone = k_first == k_last;
    for (int qi = w; qi < G; qi += kWarps) {
      float M = -CUDART_INF_F;
#pragma unroll
      for (int w2 = 0; w2 < kWarps; w2++) M = fmaxf(M, mbuf[(w2 * G + qi) * kPartStride + kD]);
      float o[4] = {0.0f, 0.0f, 0.0f, 0.0f}, l = 0.0f;
#pragma unroll
      for (int w2 = 0; w2 < kWarps; w2++) {
        const float* rec = mbuf + (w2 * G + qi) * kPartStride;
        const float mw = rec[kD];
        const float e = (mw == -CUDART_INF_F) ? 0.0f : exp2f(mw - M);
        const float4 v = *reinterpret_cast<const float4*>(rec + 4 * lane);
        o[0] += e * v.x;
        o[1] += e * v.y;
        o[2] += e * v.z;
        o[3] += e * v.w;
        l += e * rec[kD + 1];
      }
      if (alone) {
        finish_query(o, l, p.out + (static_cast<size_t>(cu.b) * p.num_kv_heads * G + cu.h * G + qi) * kD,
                     lane, p);
      } else {
        float* rec = p.part + ((unit + kc) * G + qi) * kPartStride;
        *reinterpret_cast<float4*>(rec + 4 * lane) = make_float4(o[0], o[1], o[2], o[3]);
        if (lane == 0) {
          rec[kD] = M;
          rec[kD + 1] = l;
        }
      }
    }
    if (!alone) {
      // Last CTA to arrive merges every CTA's partial of the unit.
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        int expect = 0;
        for (long long k2 = k_first; k2 <= k_last; k2++) expect += (T * k2 / C < T * (k2 + 1) / C);
        const int old = atomicAdd(p.counters + unit, 1);
        last_flag = (old == expect - 1);
        if (last_flag) p.counters[unit] = 0;  // ready for the next call
      }
      __syncthreads();
      if (last_flag) {
        __threadfence();
        for (int qi = w; qi < G; qi += kWarps) {
          float M = -CUDART_INF_F;
          for (long long k2 = k_first; k2 <= k_last; k2++) {
            if (T * k2 / C == T * (k2 + 1) / C) continue;
            M = fmaxf(M, __ldcg(p.part + ((unit + k2) * G + qi) * kPartStride + kD));
          }
          float o[4] = {0.0f, 0.0f, 0.0f, 0.0f}, l = 0.0f;
          for (long long k2 = k_first; k2 <= k_last; k2++) {
            if (T * k2 / C == T * (k2 + 1) / C) continue;
            const float* rec = p.part + ((unit + k2) * G + qi) * kPartStride;
            const float e = exp2f(__ldcg(rec + kD) - M);
            const float4 v = __ldcg(reinterpret_cast<const float4*>(rec + 4 * lane));
            o[0] += e * v.x;
            o[1] += e * v.y;
            o[2] += e * v.z;
            o[3] += e * v.w;
            l += e * __ldcg(rec + kD + 1);
          }
          finish_query(o, l,
                       p.out + (static_cast<size_t>(cu.b) * p.num_kv_heads * G + cu.h * G + qi) * kD,
                       lane, p);
        }
      }
    }
    __syncthreads();  // the merge buffer is reused by the next unit
    if (!has_next) break;
    cu = nu;
    xs = cu.U;
  }

  if (dead) {
    // Let copies still in flight land before the CTA's shared memory is released.
    for (int j = consumed + 1; j < issued; j++)
      mbar_wait_bounded(bar_s + 8 * (j % kStages), static_cast<uint32_t>((j / kStages) & 1),
                        kWaitLimitNs);
  }
}

template <int G, int SEFF>
void* kernel_ptr() {
  return reinterpret_cast<void*>(&decode_kernel<G, SEFF>);
}

void* pick_kernel(int group, int seff) {
#define KVQ_PICK(GG)                               \
  if (group == GG) {                               \
    if (seff == 16) return kernel_ptr<GG, 16>();   \
    if (seff == 32) return kernel_ptr<GG, 32>();   \
  }
  KVQ_PICK(1)
  KVQ_PICK(2)
  KVQ_PICK(4)
  KVQ_PICK(8)
#undef KVQ_PICK
  return nullptr;
}

size_t smem_bytes(int group, int max_batch) {
  size_t s = static_cast<size_t>(kWarps) * kStages * kSlotBytes;
  s += sizeof(uint64_t) * kWarps * kStages;
  s += sizeof(float) * kWarps * group * kPartStride;
  s += static_cast<size_t>(max_batch + 1) * sizeof(int32_t);
  s += 128;  // alignment slack for the ring base
  return (s + 15) & ~static_cast<size_t>(15);
}

}  // namespace

int plan_decode(int group, int page_size, int max_batch, int num_sms, DecodeLaunch* out) {
  const int seff = page_size < kTileTokens ? page_size : kTileTokens;
  void* fn = pick_kernel(group, seff);
  if (!fn) return -1;
  const size_t smem = smem_bytes(group, max_batch);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return -2;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kThreads, smem) != cudaSuccess)
    return -2;
  if (occ < 1) return -1;
  if (occ > 3) occ = 3;
  out->grid = num_sms * occ;
  out->smem = smem;
  return 0;
}

int launch_decode(const DecodeParams& p, const DecodeLaunch& L, cudaStream_t stream) {
  const int seff = p.page_size < kTileTokens ? p.page_size : kTileTokens;
  void* fn = pick_kernel(p.group, seff);
  if (!fn) return -1;
  DecodeParams q = p;
  q.total_ctas = L.grid;
  void* args[] = {&q};
  if (cudaLaunchKernel(fn, dim3(L.grid), dim3(kThreads), args, L.smem, stream) != cudaSuccess)
    return -2;
  return 0;
}

}  // namespace kvq

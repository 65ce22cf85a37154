// decode_kernel.cu -- paged GQA decode attention over the rotated INT4 cache, sm_100a.
//
// Method: "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化"
// (youngju.dev), section "KVキャッシュこそが本当のボトルネックである理由" (paged memory
// layout, regular access, fused attention execution) and section "回転のトリック —
// ブロック対角アダマール" (the rotation is orthogonal, so q.k is unchanged when both are
// rotated, and the rotation is undone exactly on the output).  Every decode step
// streams the whole cache, so the pass is HBM-bound; the design keeps the bytes moving:
//
// Split pass (decode_split_kernel).  Work is cut into tiles of 64 tokens of one
// (sequence, KV head) "unit"; tiles are numbered unit-major and warp w of the grid takes
// the contiguous tile range [w*T/W, (w+1)*T/W) (T tiles, W warps), so every warp gets
// the same number of tiles (+-1) whatever the length mix.  A warp keeps one online
// softmax state per unit it touches and writes a partial (o', m, l) per (unit, warp)
// pair to slot unit+warp of the scratch (unique along the staircase of ranges).
//
// Each warp owns a ring of 3 shared-memory slots.  One lane per page issues a 1-D bulk
// copy (cp.async.bulk, TMA engine, no multicast) of the contiguous (page, head) block --
// codes and scales together -- into the slot, completing on the slot's mbarrier; page
// ids of the tile three ahead are read while the current tile computes.
//
// Tensor cores (mma.sync m16n8k16, f16 x f16 -> f32), operands swapped so the GQA query
// group is the N = 8 side and the dequantised cache is the M = 16 side:
//   QK^T: A = K codes [16 tokens x 16 channels] (int4 -> fp16 in registers, exact),
//         B = rotated q' [16 channels x 8 columns]; the channel order inside each k16
//         step is chosen so that one thread's fragment is one 32-bit word of codes
//         (the score is a sum over channels, so any consistent order gives the same dot
//         product).  q' = q_hi + q_lo in two fp16 parts: for G <= 4 the columns hold
//         (hi, lo) of each query side by side, for G = 8 two MMAs accumulate hi and lo.
//   PV:   A = V codes transposed [16 channels x 16 tokens], built from byte permutes of
//         two token rows; B = P' [16 tokens x 8 columns] with P' = p * s_v (the V scale
//         folded into the probabilities); for G <= 4 P' is also split into hi/lo columns.
// The K scale multiplies the fp32 score of its token.  Softmax runs in the log2 domain
// (q' carries softmax_scale * log2 e) with exp2.
//
// Combine pass (decode_combine_kernel).  One warp per (sequence, query head): LSE-merge
// of the unit's partials, division by l, inverse block-diagonal FWHT across the warp
// (the orthonormal Sylvester matrix is its own inverse), fp16 store.
#include <cuda_fp16.h>
#include <math_constants.h>
#include <stdint.h>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kD = 128;
constexpr int kSlotBytes = kTileTokens * (kD + 4);  // 8448: one tile of codes + scales
constexpr int kWarps = 4;                           // warps per CTA (split pass)
constexpr int kStages = 3;                          // ring slots per warp
constexpr uint64_t kWaitLimitNs = 2000000000ull;    // bounded waits: 2 s
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ int clamp_len(int L, int cap, int32_t* status) {
  if (L < 0 || L > cap) {
    atomicOr(status, KVQ_DEV_BAD_POS_BIT);
    return L < 0 ? 0 : cap;
  }
  return L;
}

// Position of one warp in the unit-major tile sequence.
struct Cursor {
  int b;   // sequence
  int h;   // KV head
  int k;   // tile inside the unit
  int n;   // tiles in the unit
  int L;   // tokens in the sequence (clamped)
};

__device__ __forceinline__ void cursor_seek(Cursor& c, long long x, const int32_t* pre,
                                            const DecodeParams& p) {
  int lo = 0, hi = p.batch;  // pre[lo]*Hkv <= x < pre[hi]*Hkv
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<long long>(pre[mid]) * p.num_kv_heads <= x) lo = mid; else hi = mid;
  }
  c.b = lo;
  c.n = pre[lo + 1] - pre[lo];
  const long long r = x - static_cast<long long>(pre[lo]) * p.num_kv_heads;
  c.h = static_cast<int>(r / c.n);
  c.k = static_cast<int>(r % c.n);
  c.L = clamp_len(__ldg(p.seq_lens + c.b), p.max_pages_per_seq * p.page_size, p.status);
}

// Advance to the next tile.  Only called while another tile exists.
__device__ __forceinline__ void cursor_next(Cursor& c, const int32_t* pre,
                                            const DecodeParams& p) {
  if (++c.k < c.n) return;
  c.k = 0;
  if (++c.h < p.num_kv_heads) return;
  c.h = 0;
  do { ++c.b; } while (c.b < p.batch && pre[c.b + 1] == pre[c.b]);
  if (c.b < p.batch) {
    c.n = pre[c.b + 1] - pre[c.b];
    c.L = clamp_len(__ldg(p.seq_lens + c.b), p.max_pages_per_seq * p.page_size, p.status);
  }
}

// Page ids a tile needs: lane j < 4 reads the j-th page of the tile (or -1).
template <int SEFF>
__device__ __forceinline__ int tile_page_id(const Cursor& c, int lane, const DecodeParams& p) {
  const int S = p.page_size;
  const int t0 = c.k * kTileTokens;
  const int t1 = min(t0 + kTileTokens, c.L);
  int npg;
  if (S <= kTileTokens) npg = (t1 - 1) / S - t0 / S + 1;
  else npg = 1;
  if (lane >= npg) return -1;
  const int lp = t0 / S + lane;
  return __ldg(p.page_table + static_cast<size_t>(c.b) * p.max_pages_per_seq + lp);
}

// Issue the bulk copies of one tile into a ring slot (whole warp calls).
template <int SEFF>
__device__ __forceinline__ void tile_issue(const Cursor& c, int pid, uint32_t slot, uint32_t bar,
                                           int lane, uint64_t pol, const DecodeParams& p) {
  const int S = p.page_size;
  const size_t blk_bytes = static_cast<size_t>(S) * (kD + 4);
  const int t0 = c.k * kTileTokens;
  const int t1 = min(t0 + kTileTokens, c.L);
  int npg, total;
  if (S <= kTileTokens) {
    npg = (t1 - 1) / S - t0 / S + 1;
    total = npg * static_cast<int>(blk_bytes);
  } else {
    npg = 4;  // four pieces of one page
    total = kSlotBytes;
  }
  const bool need = (S <= kTileTokens) ? lane < npg : lane < 1;
  const bool bad = need && (pid < 0 || pid >= p.num_pages);
  if (__any_sync(kFull, bad) && lane == 0) atomicOr(p.status, KVQ_DEV_BAD_PAGE_BIT);
  if (bad) pid = 0;  // keep the barrier's byte count; results are flagged as invalid
  if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(total));
  __syncwarp();
  if (S <= kTileTokens) {
    if (lane < npg) {
      const uint8_t* src = p.pool_layer + (static_cast<size_t>(pid) * p.num_kv_heads + c.h) * blk_bytes;
      bulk_copy_g2s(slot + lane * static_cast<uint32_t>(blk_bytes), src,
                    static_cast<uint32_t>(blk_bytes), bar, pol);
    }
  } else {
    const int pid0 = __shfl_sync(kFull, pid, 0);
    const int o = t0 % S;  // first token of the tile inside the page
    const uint8_t* blk = p.pool_layer + (static_cast<size_t>(pid0) * p.num_kv_heads + c.h) * blk_bytes;
    if (lane == 0) bulk_copy_g2s(slot, blk + static_cast<size_t>(o) * 64, 4096, bar, pol);
    if (lane == 1)
      bulk_copy_g2s(slot + 4096, blk + static_cast<size_t>(S) * 64 + static_cast<size_t>(o) * 64, 4096, bar, pol);
    if (lane == 2)
      bulk_copy_g2s(slot + 8192, blk + static_cast<size_t>(S) * 128 + static_cast<size_t>(o) * 2, 128, bar, pol);
    if (lane == 3)
      bulk_copy_g2s(slot + 8320, blk + static_cast<size_t>(S) * 130 + static_cast<size_t>(o) * 2, 128, bar, pol);
  }
}

__device__ __forceinline__ uint32_t unpack_nib(uint32_t w, int s) {
  // s is a compile-time constant after unrolling.
  if (s == 0) return nib_lo_to_half2(w);
  if (s == 1) return nib_hi_to_half2(w);
  if (s == 2) return nib_lo_to_half2(w >> 8);
  return nib_hi_to_half2(w >> 8);
}

// Rotated, scaled q' of one query row in B-fragment order.  Thread (g, c) holds the
// row's channels [32c, 32c+32); the butterfly stages for bits 0-4 are in registers and
// bits 5, 6 are shuffles with lanes ^1, ^2 (same c-group layout as the append kernel's
// fixed stage order).  Returns hi/lo fp16 words: frag[jj][0] for k = 2c, 2c+1 and
// frag[jj][1] for k = 2c+8, 2c+9 of k-step jj.
__device__ __forceinline__ void rotate_q(const __half* qrow, bool valid, int c, int block,
                                         float cb, float qscale, uint32_t (&hi)[8][2],
                                         uint32_t (&lo)[8][2]) {
  float x[32];
  if (valid) {
    const uint4* src = reinterpret_cast<const uint4*>(qrow + 32 * c);
#pragma unroll
    for (int v = 0; v < 4; v++) {
      const uint4 u = __ldg(src + v);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
        x[8 * v + 2 * e] = f.x;
        x[8 * v + 2 * e + 1] = f.y;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; i++) x[i] = 0.0f;
  }
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
  __half xh[32], xl[32];
#pragma unroll
  for (int i = 0; i < 32; i++) {
    const float v = __fmul_rn(__fmul_rn(x[i], cb), qscale);
    xh[i] = __float2half_rn(v);
    xl[i] = __float2half_rn(__fsub_rn(v, __half2float(xh[i])));
  }
#pragma unroll
  for (int jj = 0; jj < 8; jj++) {
    const int base = 8 * (jj >> 1) + 2 * (jj & 1);
    hi[jj][0] = pack_half2(xh[base], xh[base + 4]);
    hi[jj][1] = pack_half2(xh[base + 1], xh[base + 5]);
    lo[jj][0] = pack_half2(xl[base], xl[base + 4]);
    lo[jj][1] = pack_half2(xl[base + 1], xl[base + 5]);
  }
}

template <int G>
struct SplitState {
  static constexpr int NQ = (G == 8) ? 2 : 1;  // queries owned by one thread
  uint32_t bq[8][2];                           // G<=4: packed hi|lo columns; G=8: hi
  uint32_t bl[8][2];                           // G=8: lo part
  float o[8][4];                               // PV accumulators (8 m-tiles of 16 channels)
  float m[NQ];
  float l[NQ];
};

template <int G>
__device__ __forceinline__ void state_reset(SplitState<G>& st) {
#pragma unroll
  for (int i = 0; i < 8; i++)
#pragma unroll
    for (int e = 0; e < 4; e++) st.o[i][e] = 0.0f;
#pragma unroll
  for (int qq = 0; qq < SplitState<G>::NQ; qq++) {
    st.m[qq] = -CUDART_INF_F;
    st.l[qq] = 0.0f;
  }
}

template <int G>
__device__ __forceinline__ void load_unit_q(SplitState<G>& st, const Cursor& c, int lane,
                                            const DecodeParams& p) {
  const int g = lane >> 2, cc = lane & 3;
  int qi;
  bool valid;
  if (G == 8) {
    qi = g;
    valid = true;
  } else {
    qi = g >> 1;
    valid = qi < G;
  }
  const int hq = c.h * G + (valid ? qi : 0);
  const __half* qrow = p.q + (static_cast<size_t>(c.b) * p.num_kv_heads * G + hq) * kD;
  uint32_t hi[8][2], lo[8][2];
  rotate_q(qrow, valid, cc, p.hadamard_block, p.cb, p.q_scale, hi, lo);
#pragma unroll
  for (int jj = 0; jj < 8; jj++)
#pragma unroll
    for (int e = 0; e < 2; e++) {
      if (G == 8) {
        st.bq[jj][e] = hi[jj][e];
        st.bl[jj][e] = lo[jj][e];
      } else {
        st.bq[jj][e] = (g & 1) ? lo[jj][e] : hi[jj][e];
      }
    }
}

// One 64-token tile from ring slot `slot` (shared address), ntok valid tokens.
template <int G, int SEFF>
__device__ __forceinline__ void tile_compute(SplitState<G>& st, uint32_t slot, int ntok,
                                             int lane) {
  constexpr int NQ = SplitState<G>::NQ;
  const int g = lane >> 2, c = lane & 3;
  const int tau0 = (g < 4) ? g : g + 4;  // token of A row g (QK^T)
  const int tau1 = tau0 + 4;             // token of A row g + 8
  float sc[4][NQ][2];                    // scores, log2 domain: [k-step][query][row]

#pragma unroll
  for (int j = 0; j < 4; j++) {
    const uint32_t pbase = slot + (16 * j / SEFF) * (SEFF * 132);
    const int sl = (16 * j) % SEFF;
    const uint32_t kb = pbase + sl * 64;
    const uint32_t skb = pbase + SEFF * 128 + sl * 2;
    const uint4 ka = lds_128(kb + tau0 * 64 + 16 * c);
    const uint4 kc = lds_128(kb + tau1 * 64 + 16 * c);
    const uint32_t kaw[4] = {ka.x, ka.y, ka.z, ka.w};
    const uint32_t kcw[4] = {kc.x, kc.y, kc.z, kc.w};
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int jj = 0; jj < 8; jj++) {
      const int w = jj >> 1, s0 = 2 * (jj & 1);
      const uint32_t a0 = unpack_nib(kaw[w], s0);
      const uint32_t a1 = unpack_nib(kcw[w], s0);
      const uint32_t a2 = unpack_nib(kaw[w], s0 + 1);
      const uint32_t a3 = unpack_nib(kcw[w], s0 + 1);
      mma_16816(acc, a0, a1, a2, a3, st.bq[jj][0], st.bq[jj][1]);
      if (G == 8) mma_16816(acc, a0, a1, a2, a3, st.bl[jj][0], st.bl[jj][1]);
    }
    const float sk0 = __half2float(__ushort_as_half(lds_u16(skb + tau0 * 2)));
    const float sk1 = __half2float(__ushort_as_half(lds_u16(skb + tau1 * 2)));
    const bool v0 = 16 * j + tau0 < ntok, v1 = 16 * j + tau1 < ntok;
    if (G == 8) {
      sc[j][0][0] = v0 ? acc[0] * sk0 : -CUDART_INF_F;
      sc[j][NQ - 1][0] = v0 ? acc[1] * sk0 : -CUDART_INF_F;
      sc[j][0][1] = v1 ? acc[2] * sk1 : -CUDART_INF_F;
      sc[j][NQ - 1][1] = v1 ? acc[3] * sk1 : -CUDART_INF_F;
    } else {
      sc[j][0][0] = v0 ? (acc[0] + acc[1]) * sk0 : -CUDART_INF_F;
      sc[j][0][1] = v1 ? (acc[2] + acc[3]) * sk1 : -CUDART_INF_F;
    }
  }

  // Online softmax over the tile (log2 domain).
  float alpha[NQ];
  bool rescale = false;
#pragma unroll
  for (int qq = 0; qq < NQ; qq++) {
    float mx = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < 4; j++) mx = fmaxf(mx, fmaxf(sc[j][qq][0], sc[j][qq][1]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
    const float mnew = fmaxf(st.m[qq], mx);
    alpha[qq] = exp2f(st.m[qq] - mnew);
    rescale |= alpha[qq] != 1.0f;
    st.m[qq] = mnew;
    float ps = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; j++)
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
      if (G == 8) {
        st.o[i][0] *= alpha[0];
        st.o[i][2] *= alpha[0];
        st.o[i][1] *= alpha[NQ - 1];
        st.o[i][3] *= alpha[NQ - 1];
      } else {
#pragma unroll
        for (int e = 0; e < 4; e++) st.o[i][e] *= alpha[0];
      }
    }
  }

  // PV.
  const int srcA = 4 * c + (g >> 1);
  const int srcB = srcA + 16;
  const bool bzero = (G < 4) && ((g >> 1) >= G);
#pragma unroll
  for (int j = 0; j < 4; j++) {
    const uint32_t pbase = slot + (16 * j / SEFF) * (SEFF * 132);
    const int sl = (16 * j) % SEFF;
    const uint32_t vb = pbase + SEFF * 64 + sl * 64;
    const uint32_t svb = pbase + SEFF * 130 + sl * 2;
    const float sv0 = __half2float(__ushort_as_half(lds_u16(svb + tau0 * 2)));
    const float sv1 = __half2float(__ushort_as_half(lds_u16(svb + tau1 * 2)));
    const bool v0 = 16 * j + tau0 < ntok, v1 = 16 * j + tau1 < ntok;
    uint32_t x0, x1;
    if (G == 8) {
      const float p00 = v0 ? sc[j][0][0] * sv0 : 0.0f, p01 = v1 ? sc[j][0][1] * sv1 : 0.0f;
      const float p10 = v0 ? sc[j][1][0] * sv0 : 0.0f, p11 = v1 ? sc[j][1][1] * sv1 : 0.0f;
      x0 = pack_half2(__float2half_rn(p00), __float2half_rn(p01));
      x1 = pack_half2(__float2half_rn(p10), __float2half_rn(p11));
    } else {
      const float p0 = v0 ? sc[j][0][0] * sv0 : 0.0f, p1 = v1 ? sc[j][0][1] * sv1 : 0.0f;
      const __half h0 = __float2half_rn(p0), h1 = __float2half_rn(p1);
      x0 = pack_half2(h0, h1);
      x1 = pack_half2(__float2half_rn(p0 - __half2float(h0)), __float2half_rn(p1 - __half2float(h1)));
    }
    const uint32_t yA0 = __shfl_sync(kFull, x0, srcA), yA1 = __shfl_sync(kFull, x1, srcA);
    const uint32_t yB0 = __shfl_sync(kFull, x0, srcB), yB1 = __shfl_sync(kFull, x1, srcB);
    uint32_t b0 = (g & 1) ? yA1 : yA0;
    uint32_t b1 = (g & 1) ? yB1 : yB0;
    if (bzero) b0 = b1 = 0u;

    // V rows of tokens c, c+4, c+8, c+12; this thread's channels [16g, 16g+16).
    const uint2 t0 = lds_64(vb + (c + 0) * 64 + 8 * g);
    const uint2 t1 = lds_64(vb + (c + 4) * 64 + 8 * g);
    const uint2 t2 = lds_64(vb + (c + 8) * 64 + 8 * g);
    const uint2 t3 = lds_64(vb + (c + 12) * 64 + 8 * g);
    const uint32_t w0[2] = {t0.x, t0.y}, w1[2] = {t1.x, t1.y};
    const uint32_t w2[2] = {t2.x, t2.y}, w3[2] = {t3.x, t3.y};
#pragma unroll
    for (int wi = 0; wi < 2; wi++)
#pragma unroll
      for (int ph = 0; ph < 2; ph++) {
        const uint32_t sel = ph ? 0x7632u : 0x5410u;
        const uint32_t r01 = prmt(w0[wi], w1[wi], sel);
        const uint32_t r23 = prmt(w2[wi], w3[wi], sel);
#pragma unroll
        for (int odd = 0; odd < 2; odd++) {
          const int i = 4 * wi + 2 * ph + odd;  // m-tile: channels 16g+2i, 16g+2i+1
          const int s = 2 * odd;
          mma_16816(st.o[i], unpack_nib(r01, s), unpack_nib(r01, s + 1), unpack_nib(r23, s),
                    unpack_nib(r23, s + 1), b0, b1);
        }
      }
  }
}

// Write the warp's partial for unit u to slot u + wid.
template <int G>
__device__ __forceinline__ void state_flush(const SplitState<G>& st, long long slot_idx, int lane,
                                            const DecodeParams& p) {
  constexpr int NQ = SplitState<G>::NQ;
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int qq = 0; qq < NQ; qq++) {
    float l = st.l[qq];
    l += __shfl_xor_sync(kFull, l, 4);
    l += __shfl_xor_sync(kFull, l, 8);
    l += __shfl_xor_sync(kFull, l, 16);
    int qi;
    bool own;
    if (G == 8) { qi = 2 * c + qq; own = true; }
    else { qi = c; own = c < G; }
    if (!own) continue;
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; i++) {
      if (G == 8) {
        v[2 * i] = st.o[i][qq];
        v[2 * i + 1] = st.o[i][2 + qq];
      } else {
        v[2 * i] = st.o[i][0] + st.o[i][1];
        v[2 * i + 1] = st.o[i][2] + st.o[i][3];
      }
    }
    float* rec = p.part + (static_cast<size_t>(slot_idx) * G + qi) * kPartStride;
    float4* dst = reinterpret_cast<float4*>(rec + 16 * g);
#pragma unroll
    for (int e = 0; e < 4; e++) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    if (g == 0) {
      rec[kD] = st.m[qq];
      rec[kD + 1] = l;
    }
  }
}

template <int G, int SEFF>
__global__ void __launch_bounds__(kWarps * 32) decode_split_kernel(DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  // Bulk copies need 16-byte aligned destinations; align the ring to 128 bytes (the
  // allocation carries 128 spare bytes for this).
  uint8_t* smem = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * kSlotBytes);
  int32_t* pre = reinterpret_cast<int32_t*>(bars + kWarps * kStages);
  __shared__ int warp_sum[kWarps];
  __shared__ int running;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cap = p.max_pages_per_seq * p.page_size;

  // Tiles per sequence -> exclusive prefix pre[0..batch] (block-wide scan).
  if (tid == 0) running = 0;
  __syncthreads();
  for (int base = 0; base < p.batch; base += kWarps * 32) {
    const int i = base + tid;
    int n = 0;
    if (i < p.batch) n = (clamp_len(__ldg(p.seq_lens + i), cap, p.status) + kTileTokens - 1) / kTileTokens;
    int incl = n;
#pragma unroll
    for (int d = 1; d < 32; d *= 2) {
      const int y = __shfl_up_sync(kFull, incl, d);
      if (lane >= d) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int before = running;
    for (int w2 = 0; w2 < warp; w2++) before += warp_sum[w2];
    if (i < p.batch) pre[i] = before + incl - n;
    __syncthreads();
    if (tid == kWarps * 32 - 1) running = before + incl;
    __syncthreads();
  }
  if (tid == 0) pre[p.batch] = running;
  __syncthreads();
  if (blockIdx.x == 0)
    for (int i = tid; i <= p.batch; i += kWarps * 32) p.tile_prefix[i] = pre[i];

  const long long T = static_cast<long long>(pre[p.batch]) * p.num_kv_heads;
  const long long W = p.total_warps;
  const long long wid = static_cast<long long>(blockIdx.x) * kWarps + warp;
  const long long x0 = T * wid / W, x1 = T * (wid + 1) / W;
  if (x0 >= x1) return;
  const long long count = x1 - x0;

  const uint32_t ring_s = smem_addr(ring + warp * kStages * kSlotBytes);
  const uint32_t bar_s = smem_addr(bars + warp * kStages);
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; s++) mbar_init(bar_s + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_policy_evict_first();

  Cursor pc, cc;
  cursor_seek(pc, x0, pre, p);
  cc = pc;
  const long long npro = count < kStages ? count : kStages;
  for (long long s = 0; s < npro; s++) {
    const int pid = tile_page_id<SEFF>(pc, lane, p);
    tile_issue<SEFF>(pc, pid, ring_s + static_cast<uint32_t>(s) * kSlotBytes,
                     bar_s + 8 * static_cast<uint32_t>(s), lane, pol, p);
    if (s + 1 < count) cursor_next(pc, pre, p);
  }

  SplitState<G> st;
  int cur_b = -1, cur_h = -1;
  bool timed_out = false;
  long long i = 0;
  for (; i < count; i++) {
    const int s = static_cast<int>(i % kStages);
    const uint32_t parity = static_cast<uint32_t>((i / kStages) & 1);
    const bool more = i + kStages < count;
    const int pid_next = more ? tile_page_id<SEFF>(pc, lane, p) : -1;

    if (cc.b != cur_b || cc.h != cur_h) {
      if (cur_b >= 0)
        state_flush<G>(st, static_cast<long long>(cur_b) * p.num_kv_heads + cur_h + wid, lane, p);
      cur_b = cc.b;
      cur_h = cc.h;
      state_reset<G>(st);
      load_unit_q<G>(st, cc, lane, p);
    }
    if (!mbar_wait_bounded(bar_s + 8 * s, parity, kWaitLimitNs)) {
      timed_out = true;
      break;
    }
    const int ntok = min(kTileTokens, cc.L - cc.k * kTileTokens);
    tile_compute<G, SEFF>(st, ring_s + static_cast<uint32_t>(s) * kSlotBytes, ntok, lane);
    __syncwarp();
    if (more) {
      fence_proxy_async_smem();
      tile_issue<SEFF>(pc, pid_next, ring_s + static_cast<uint32_t>(s) * kSlotBytes,
                       bar_s + 8 * s, lane, pol, p);
      if (i + kStages + 1 < count) cursor_next(pc, pre, p);
    }
    if (i + 1 < count) cursor_next(cc, pre, p);
  }
  if (timed_out) {
    if (lane == 0) atomicOr(p.status, KVQ_DEV_TIMEOUT_BIT);
    // Let copies still in flight land before the CTA's shared memory is released.
    const long long issued = count < i + kStages ? count : i + kStages;
    for (long long j = i + 1; j < issued; j++)
      mbar_wait_bounded(bar_s + 8 * static_cast<uint32_t>(j % kStages),
                        static_cast<uint32_t>((j / kStages) & 1), kWaitLimitNs);
    return;
  }
  if (cur_b >= 0)
    state_flush<G>(st, static_cast<long long>(cur_b) * p.num_kv_heads + cur_h + wid, lane, p);
}

// One warp per (sequence, query head).
__global__ void __launch_bounds__(128) decode_combine_kernel(DecodeParams p) {
  const int lane = threadIdx.x & 31;
  const long long gw = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int hq_count = p.num_kv_heads * p.group;
  if (gw >= static_cast<long long>(p.batch) * hq_count) return;
  const int b = static_cast<int>(gw / hq_count), hq = static_cast<int>(gw % hq_count);
  const int h = hq / p.group, qi = hq % p.group;
  const int32_t* pre = p.tile_prefix;
  const int n = pre[b + 1] - pre[b];
  __half* orow = p.out + (static_cast<size_t>(b) * hq_count + hq) * kD + 4 * lane;
  if (n == 0) {
    *reinterpret_cast<uint2*>(orow) = make_uint2(0u, 0u);
    return;
  }
  const long long T = static_cast<long long>(pre[p.batch]) * p.num_kv_heads;
  const long long W = p.total_warps;
  const long long u0 = static_cast<long long>(pre[b]) * p.num_kv_heads + static_cast<long long>(h) * n;
  const long long wf = ((u0 + 1) * W - 1) / T;
  const long long wl = ((u0 + n) * W - 1) / T;
  const long long unit = static_cast<long long>(b) * p.num_kv_heads + h;

  // Warps wf..wl cover the unit's tiles; a warp whose range is empty (more warps than
  // tiles) wrote nothing and is skipped.
  float M = -CUDART_INF_F;
  for (long long w = wf; w <= wl; w++) {
    if (T * w / W == T * (w + 1) / W) continue;
    M = fmaxf(M, p.part[((unit + w) * p.group + qi) * kPartStride + kD]);
  }
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f}, lsum = 0.0f;
  for (long long w = wf; w <= wl; w++) {
    if (T * w / W == T * (w + 1) / W) continue;
    const float* rec = p.part + ((unit + w) * p.group + qi) * kPartStride;
    const float e = exp2f(rec[kD] - M);
    const float4 o = *reinterpret_cast<const float4*>(rec + 4 * lane);
    acc[0] += e * o.x;
    acc[1] += e * o.y;
    acc[2] += e * o.z;
    acc[3] += e * o.w;
    lsum += e * rec[kD + 1];
  }
  float x[4];
#pragma unroll
  for (int e = 0; e < 4; e++) x[e] = __fdiv_rn(acc[e], lsum);
  // Inverse rotation: stages h = 1, 2 in registers, h = 4 .. 64 across lanes.
  const int block = p.hadamard_block;
  if (1 < block) {
    float a = x[0], c = x[1]; x[0] = a + c; x[1] = a - c;
    a = x[2]; c = x[3]; x[2] = a + c; x[3] = a - c;
  }
  if (2 < block) {
    float a = x[0], c = x[2]; x[0] = a + c; x[2] = a - c;
    a = x[1]; c = x[3]; x[1] = a + c; x[3] = a - c;
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
  *reinterpret_cast<uint2*>(orow) = make_uint2(lo, hi);
}

template <int G, int SEFF>
void* split_kernel_ptr() {
  return reinterpret_cast<void*>(&decode_split_kernel<G, SEFF>);
}

void* pick_split_kernel(int group, int seff) {
#define KVQ_PICK(GG)                                   \
  if (group == GG) {                                   \
    if (seff == 16) return split_kernel_ptr<GG, 16>(); \
    if (seff == 32) return split_kernel_ptr<GG, 32>(); \
    if (seff == 64) return split_kernel_ptr<GG, 64>(); \
  }
  KVQ_PICK(1)
  KVQ_PICK(2)
  KVQ_PICK(4)
  KVQ_PICK(8)
#undef KVQ_PICK
  return nullptr;
}

size_t split_smem_bytes(int batch) {
  size_t s = static_cast<size_t>(kWarps) * kStages * kSlotBytes + sizeof(uint64_t) * kWarps * kStages;
  s += static_cast<size_t>(batch + 1) * sizeof(int32_t);
  s += 128;  // alignment slack for the ring base
  return (s + 15) & ~static_cast<size_t>(15);
}

}  // namespace

int max_decode_warps(int num_sms) { return num_sms * 2 * kWarps; }

int plan_decode(int group, int page_size, int batch, int num_sms, DecodeLaunch* out) {
  const int seff = page_size < kTileTokens ? page_size : kTileTokens;
  void* fn = pick_split_kernel(group, seff);
  if (!fn) return -1;
  const size_t smem = split_smem_bytes(batch);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return -2;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kWarps * 32, smem) != cudaSuccess)
    return -2;
  if (occ < 1) return -1;
  if (occ > 2) occ = 2;
  out->grid = num_sms * occ;
  out->warps = out->grid * kWarps;
  out->smem = smem;
  return 0;
}

int launch_decode(const DecodeParams& p, const DecodeLaunch& L, cudaStream_t stream) {
  const int seff = p.page_size < kTileTokens ? p.page_size : kTileTokens;
  void* fn = pick_split_kernel(p.group, seff);
  if (!fn) return -1;
  DecodeParams q = p;
  q.total_warps = L.warps;
  void* args[] = {&q};
  if (cudaLaunchKernel(fn, dim3(L.grid), dim3(kWarps * 32), args, L.smem, stream) != cudaSuccess)
    return -2;
  const long long rows = static_cast<long long>(p.batch) * p.num_kv_heads * p.group;
  if (rows > 0) {
    decode_combine_kernel<<<static_cast<unsigned>((rows + 3) / 4), 128, 0, stream>>>(q);
    if (cudaGetLastError() != cudaSuccess) return -2;
  }
  return 0;
}

}  // namespace kvq

// kvq_internal.h -- parameter blocks shared by the host code and the kernels of libkvq.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvq.h"

namespace kvq {

// Descriptor validation shared by every entry point that takes a kvq_desc: true when the
// geometry is one the kernels implement; otherwise *why is KVQ_EINVAL (a null descriptor,
// a non-positive size) or KVQ_EUNSUPPORTED (a shape outside the kernels).
bool desc_valid(const kvq_desc* d, int* why);
// Bytes of one token row of a (page, head) block (132 INT4, 144 NVFP4) and of one layer of
// the pool; desc_valid(d) must hold.
size_t desc_row_bytes(const kvq_desc* d);
size_t desc_layer_bytes(const kvq_desc* d);

// Device status bits (same values as KVQ_DEV_* in include/kvq.h).
constexpr int KVQ_DEV_BAD_PAGE_BIT = 1;
constexpr int KVQ_DEV_BAD_POS_BIT = 2;
constexpr int KVQ_DEV_TIMEOUT_BIT = 4;

struct AppendParams {
  uint8_t* pool_layer;            // block(0, 0) of the layer
  const __half* k;                // [T][Hkv][128]
  const __half* v;                // [T][Hkv][128]
  const int32_t* cu_new_tokens;   // [batch+1]
  const int32_t* seq_lens;        // [batch], before the append
  const int32_t* page_table;      // [batch][max_pages_per_seq]
  int32_t* status;                // device status word
  int batch;
  int total_new_tokens;
  int num_kv_heads;
  int num_pages;
  int page_size;
  int max_pages_per_seq;
  float cb;                       // fp32 nearest 1/sqrt(hadamard_block)
  int fp4;                        // 1: NVFP4 rows (E2M1 codes, E4M3 scale per 16 channels)
  int page_shift;                 // log2(page_size)
  // n / num_kv_heads for 0 <= n < 2^31 as umulhi(2n, heads_magic) >> heads_shift
  uint32_t heads_magic;
  int heads_shift;
};

// Tokens per decode tile (one shared-memory ring slot per tile).
constexpr int kTileTokens = 32;
// fp32 words per (partial, query) record in the split scratch: o'[128], m, l, 2 pad.
constexpr int kPartStride = 132;
// Warps per decode CTA; each (unit, CTA) partial slot holds one record per warp.
constexpr int kDecodeWarps = 4;

struct DecodeParams {
  const uint8_t* pool_layer;      // block(0, 0) of the layer
  const __half* q;                // [batch][Hq][128]
  const int32_t* seq_lens;        // [batch], tokens to attend
  const int32_t* page_table;      // [batch][max_pages_per_seq]
  __half* out;                    // [batch][Hq][128]
  float* part;                    // per-(unit, CTA) partials [slots][G][kPartStride]
  int32_t* counters;              // [max_batch * Hkv] arrival counters, zero between calls
  int32_t* status;
  int batch;
  int num_kv_heads;
  int group;                      // G = Hq / Hkv
  int num_pages;
  int page_size;
  int page_shift;                 // log2(page_size)
  int max_pages_per_seq;
  int hadamard_block;
  float q_scale;                  // softmax_scale * log2(e)
  float cb;                       // fp32 nearest 1/sqrt(hadamard_block)
  int total_ctas;                 // C: CTAs in the grid
  // Fused one-token append (null for a plain decode): the new K and V rows [batch][Hkv][128]
  // are rotated, quantised and stored at position seq_lens[b], and the decode runs over
  // seq_lens[b] + 1 tokens (the pool is then written through pool_layer).
  const __half* k_new;
  const __half* v_new;
  int fp4;                        // 1: NVFP4 cache (host-side kernel choice)
};

struct PrefillParams {
  const uint8_t* pool_layer;      // block(0, 0) of the layer
  const __half* q;                // [total_q][Hq][128], chunks concatenated by sequence
  const int32_t* cu_q;            // [batch+1] chunk offsets
  const int32_t* seq_lens;        // [batch] tokens cached, the chunk included
  const int32_t* page_table;      // [batch][max_pages_per_seq]
  __half* out;                    // [total_q][Hq][128]
  int32_t* status;
  int batch;
  int num_kv_heads;
  int group;
  int num_pages;
  int page_size;
  int page_shift;
  int max_pages_per_seq;
  int hadamard_block;
  float q_scale;                  // softmax_scale * log2(e)
  float cb;
  int total_q;                    // rows of q and out
  int fp4;                        // 1: NVFP4 cache
};

// Host-side launchers (return 0 on success, <0 on an unsupported shape or a launch
// error).
int launch_append(const AppendParams& p, int block, int num_sms, cudaStream_t stream);
// Chunked prefill on the 5th-generation tensor cores (INT4 and NVFP4 caches).
int launch_prefill_tc(const PrefillParams& p, int total_q, cudaStream_t stream);

struct DecodeLaunch {
  int grid;          // CTAs (a multiple of the SM count)
  size_t smem;       // dynamic shared memory per CTA
};
// Shape of the decode pass for a batch capacity (grid sized to fill every SM).
int plan_decode(int group, int page_size, int max_batch, int num_sms, int fp4, DecodeLaunch* out);
int launch_decode(const DecodeParams& p, const DecodeLaunch& L, cudaStream_t stream);

}  // namespace kvq

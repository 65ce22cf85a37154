// kvq_api.cu -- host side of the C ABI declared in include/kvq.h: argument checks,
// the deterministic page allocator, memory ownership, and kernel launches.
//
// Sources: "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化"
// (youngju.dev): fixed-size paged KV blocks plus a page table (section
// "KVキャッシュこそが本当のボトルネックである理由"), a fused rotate-quantise-append kernel
// integrated with the paged layout (section "システムこそが設計である — 融合カーネル").
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include <new>

#include "../../include/kvq.h"
#include "kvq_internal.h"

struct kvq_cache {
  kvq_desc d;
  uint8_t* pool;
  size_t pool_bytes;
  bool own_pool;
  void* scratch;             // one allocation: status word, unit counters, partials
  int32_t* status;
  int32_t* counters;
  float* part;
  int device;
  int num_sms;
  kvq::DecodeLaunch launch;  // split-pass shape, fixed for the handle
  float cb;
};

namespace kvq {

bool desc_valid(const kvq_desc* d, int* why) {
  *why = KVQ_EINVAL;
  if (!d) return false;
  if (d->num_layers < 1 || d->num_kv_heads < 1 || d->num_q_heads < 1 || d->num_pages < 1 ||
      d->max_batch < 1 || d->max_pages_per_seq < 1 || d->page_size < 1 || d->head_dim < 1 ||
      d->hadamard_block < 1)
    return false;
  *why = KVQ_EUNSUPPORTED;
  if (d->num_q_heads % d->num_kv_heads) return false;
  const int g = d->num_q_heads / d->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return false;
  if (d->head_dim != 128) return false;
  const int hb = d->hadamard_block;
  if (hb != 1 && hb != 32 && hb != 64 && hb != 128) return false;  // 1: plain INT4, no rotation
  const int S = d->page_size;
  if (S != 16 && S != 32 && S != 64 && S != 128 && S != 256) return false;
  if (d->kv_format != KVQ_FORMAT_INT4 && d->kv_format != KVQ_FORMAT_NVFP4) return false;
  if (d->max_batch > 4096) return false;
  if (static_cast<long long>(d->max_pages_per_seq) * S > (1LL << 30)) return false;
  if (static_cast<long long>(d->max_batch) * d->max_pages_per_seq > (1LL << 31) - 1) return false;
  // The decode kernel numbers 32-token tiles of all (sequence, KV head) pairs in 32 bits.
  const long long tiles_per_seq = (static_cast<long long>(d->max_pages_per_seq) * S + 31) / 32;
  if (static_cast<long long>(d->max_batch) * d->num_kv_heads * tiles_per_seq >= (1LL << 30))
    return false;
  *why = KVQ_OK;
  return true;
}

// K and V codes, then the scales (one fp16 each for INT4; one E4M3 per 16 channels each
// for NVFP4).
size_t desc_row_bytes(const kvq_desc* d) {
  return static_cast<size_t>(d->head_dim) +
         (d->kv_format == KVQ_FORMAT_NVFP4 ? static_cast<size_t>(d->head_dim) / 8 : 4);
}

size_t desc_layer_bytes(const kvq_desc* d) {
  return static_cast<size_t>(d->num_pages) * static_cast<size_t>(d->num_kv_heads) *
         static_cast<size_t>(d->page_size) * desc_row_bytes(d);
}

}  // namespace kvq

namespace {

bool desc_ok(const kvq_desc* d, int* why) { return kvq::desc_valid(d, why); }

size_t pool_bytes_of(const kvq_desc* d) {
  return static_cast<size_t>(d->num_layers) * kvq::desc_layer_bytes(d);
}

// fp32 value nearest 1/sqrt(b) (b = 32, 64, 128).
float hadamard_scale(int b) { return static_cast<float>(1.0 / sqrt(static_cast<double>(b))); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

}  // namespace

extern "C" {

const char* kvq_status_string(int s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_EINVAL: return "invalid argument";
    case KVQ_EUNSUPPORTED: return "unsupported shape";
    case KVQ_ENOPAGES: return "not enough pages";
    case KVQ_ECUDA: return "CUDA runtime error";
    default: return "unknown status";
  }
}

size_t kvq_pool_bytes(const kvq_desc* d) {
  int why;
  if (!desc_ok(d, &why)) return 0;
  return pool_bytes_of(d);
}

int kvq_assign_pages(const kvq_desc* d, int32_t batch, const int32_t* capacity_tokens,
                     const int32_t* page_order, int32_t* page_table) {
  int why;
  if (!desc_ok(d, &why)) return why;
  if (batch < 0 || batch > d->max_batch) return KVQ_EINVAL;
  if (batch == 0) return KVQ_OK;
  if (!capacity_tokens || !page_table) return KVQ_EINVAL;
  const int S = d->page_size, mp = d->max_pages_per_seq;
  int next = 0;  // next position in the page order
  for (int b = 0; b < batch; b++) {
    const int cap = capacity_tokens[b];
    if (cap < 0) return KVQ_EINVAL;
    const long long need = (static_cast<long long>(cap) + S - 1) / S;
    if (need > mp) return KVQ_ENOPAGES;
    int32_t* row = page_table + static_cast<size_t>(b) * mp;
    for (int p = 0; p < mp; p++) {
      if (p >= need) {
        row[p] = -1;
        continue;
      }
      if (next >= d->num_pages) return KVQ_ENOPAGES;
      const int32_t page = page_order ? page_order[next] : next;
      if (page < 0 || page >= d->num_pages) return KVQ_EINVAL;
      row[p] = page;
      next++;
    }
  }
  return KVQ_OK;
}

int kvq_alloc_pages(const kvq_desc* d, void* dev_pool, size_t pool_bytes, int32_t batch,
                    const int32_t* capacity_tokens, const int32_t* page_order,
                    int32_t* page_table, kvq_cache** out) {
  if (!out) return KVQ_EINVAL;
  *out = nullptr;
  int why;
  if (!desc_ok(d, &why)) return why;
  if (batch < 0 || batch > d->max_batch) return KVQ_EINVAL;
  const size_t need = pool_bytes_of(d);
  if (dev_pool && (pool_bytes < need || !aligned16(dev_pool))) return KVQ_EINVAL;
  if (batch > 0) {
    const int rc = kvq_assign_pages(d, batch, capacity_tokens, page_order, page_table);
    if (rc != KVQ_OK) return rc;
  }

  kvq_cache* c = new (std::nothrow) kvq_cache();
  if (!c) return KVQ_ECUDA;
  c->d = *d;
  c->cb = hadamard_scale(d->hadamard_block);
  if (cudaGetDevice(&c->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) !=
          cudaSuccess) {
    delete c;
    return KVQ_ECUDA;
  }
  const int g = d->num_q_heads / d->num_kv_heads;
  if (kvq::plan_decode(g, d->page_size, d->max_batch, c->num_sms,
                       d->kv_format == KVQ_FORMAT_NVFP4, &c->launch) != 0) {
    delete c;
    return KVQ_ECUDA;
  }
  // Scratch: status word (padded to 256 B), one arrival counter per unit (zero between
  // calls; the decode kernel resets what it uses), and the per-(unit, CTA, warp) partials
  // [(max_batch * Hkv + grid) * kDecodeWarps * G * kPartStride] fp32.
  const size_t units = static_cast<size_t>(d->max_batch) * d->num_kv_heads;
  const size_t counter_bytes = (units * 4 + 255) & ~size_t(255);
  const size_t slots = (units + static_cast<size_t>(c->launch.grid)) * kvq::kDecodeWarps;
  const size_t part_bytes = slots * g * kvq::kPartStride * sizeof(float);
  if (cudaMalloc(&c->scratch, 256 + counter_bytes + part_bytes) != cudaSuccess) {
    delete c;
    return KVQ_ECUDA;
  }
  c->status = static_cast<int32_t*>(c->scratch);
  c->counters = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(c->scratch) + 256);
  c->part = reinterpret_cast<float*>(static_cast<uint8_t*>(c->scratch) + 256 + counter_bytes);
  if (cudaMemset(c->scratch, 0, 256 + counter_bytes) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(c->scratch);
    delete c;
    return KVQ_ECUDA;
  }
  if (dev_pool) {
    c->pool = static_cast<uint8_t*>(dev_pool);
    c->pool_bytes = pool_bytes;
    c->own_pool = false;
  } else {
    void* p = nullptr;
    if (cudaMalloc(&p, need) != cudaSuccess) {
      cudaFree(c->scratch);
      delete c;
      return KVQ_ECUDA;
    }
    c->pool = static_cast<uint8_t*>(p);
    c->pool_bytes = need;
    c->own_pool = true;
  }
  *out = c;
  return KVQ_OK;
}

int kvq_rotate_quant_append(kvq_cache* c, int32_t layer, const void* k, const void* v,
                            const int32_t* cu_new_tokens, const int32_t* seq_lens,
                            const int32_t* page_table, int32_t batch, int32_t total_new_tokens,
                            void* stream) {
  if (!c) return KVQ_EINVAL;
  if (layer < 0 || layer >= c->d.num_layers) return KVQ_EINVAL;
  if (batch < 0 || batch > c->d.max_batch || total_new_tokens < 0) return KVQ_EINVAL;
  if (total_new_tokens == 0) return KVQ_OK;
  if (batch == 0) return KVQ_EINVAL;
  if (!k || !v || !cu_new_tokens || !seq_lens || !page_table) return KVQ_EINVAL;
  if (!aligned32(k) || !aligned32(v)) return KVQ_EINVAL;  // 256-bit loads
  kvq::AppendParams p;
  const size_t layer_bytes = pool_bytes_of(&c->d) / c->d.num_layers;
  p.pool_layer = c->pool + static_cast<size_t>(layer) * layer_bytes;
  p.k = static_cast<const __half*>(k);
  p.v = static_cast<const __half*>(v);
  p.cu_new_tokens = cu_new_tokens;
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.status = c->status;
  p.batch = batch;
  p.total_new_tokens = total_new_tokens;
  p.num_kv_heads = c->d.num_kv_heads;
  p.num_pages = c->d.num_pages;
  p.page_size = c->d.page_size;
  p.max_pages_per_seq = c->d.max_pages_per_seq;
  p.cb = c->cb;
  p.fp4 = c->d.kv_format == KVQ_FORMAT_NVFP4;
  p.page_shift = __builtin_ctz(static_cast<unsigned>(c->d.page_size));
  // Division by an invariant integer (Granlund and Montgomery, "Division by invariant
  // integers using multiplication", 1994, Theorem 4.2 with N = 31): for l = ceil(log2 d)
  // and m = ceil(2^(31 + l) / d), floor(n * m / 2^(31 + l)) = floor(n / d) for every
  // 0 <= n < 2^31, and m < 2^32.
  {
    const unsigned d = static_cast<unsigned>(c->d.num_kv_heads);
    int l = 0;
    while ((1ull << l) < d) l++;
    p.heads_magic = static_cast<uint32_t>(((1ull << (31 + l)) + d - 1) / d);
    p.heads_shift = l;
  }
  const int rc = kvq::launch_append(p, c->d.hadamard_block, c->num_sms, static_cast<cudaStream_t>(stream));
  if (rc == -1) return KVQ_EUNSUPPORTED;
  return rc == 0 ? KVQ_OK : KVQ_ECUDA;
}

namespace {

// Shared by the decode and the fused append + decode calls.
int decode_common(kvq_cache* c, int32_t layer, const void* k_new, const void* v_new, const void* q,
                  const int32_t* seq_lens, const int32_t* page_table, int32_t batch,
                  float softmax_scale, void* out, void* stream) {
  if (!c) return KVQ_EINVAL;
  if (layer < 0 || layer >= c->d.num_layers) return KVQ_EINVAL;
  if (batch < 0 || batch > c->d.max_batch) return KVQ_EINVAL;
  if (!(softmax_scale >= 0.0f) || isinf(softmax_scale)) return KVQ_EINVAL;
  if (batch == 0) return KVQ_OK;
  if (!q || !seq_lens || !page_table || !out) return KVQ_EINVAL;
  if (!aligned16(q) || !aligned16(out)) return KVQ_EINVAL;
  kvq::DecodeParams p;
  const size_t layer_bytes = pool_bytes_of(&c->d) / c->d.num_layers;
  p.pool_layer = c->pool + static_cast<size_t>(layer) * layer_bytes;
  p.q = static_cast<const __half*>(q);
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.out = static_cast<__half*>(out);
  p.part = c->part;
  p.counters = c->counters;
  p.status = c->status;
  p.batch = batch;
  p.num_kv_heads = c->d.num_kv_heads;
  p.group = c->d.num_q_heads / c->d.num_kv_heads;
  p.num_pages = c->d.num_pages;
  p.page_size = c->d.page_size;
  p.page_shift = __builtin_ctz(static_cast<unsigned>(c->d.page_size));
  p.max_pages_per_seq = c->d.max_pages_per_seq;
  p.hadamard_block = c->d.hadamard_block;
  const double sm = softmax_scale == 0.0f ? 1.0 / sqrt(static_cast<double>(c->d.head_dim))
                                          : static_cast<double>(softmax_scale);
  p.q_scale = static_cast<float>(sm * 1.4426950408889634);  // log2(e)
  p.cb = c->cb;
  p.total_ctas = c->launch.grid;
  p.k_new = static_cast<const __half*>(k_new);
  p.v_new = static_cast<const __half*>(v_new);
  p.fp4 = c->d.kv_format == KVQ_FORMAT_NVFP4;
  const int rc = kvq::launch_decode(p, c->launch, static_cast<cudaStream_t>(stream));
  if (rc == -1) return KVQ_EUNSUPPORTED;
  return rc == 0 ? KVQ_OK : KVQ_ECUDA;
}

}  // namespace

int kvq_decode_attention(kvq_cache* c, int32_t layer, const void* q, const int32_t* seq_lens,
                         const int32_t* page_table, int32_t batch, float softmax_scale, void* out,
                         void* stream) {
  return decode_common(c, layer, nullptr, nullptr, q, seq_lens, page_table, batch, softmax_scale,
                       out, stream);
}

int kvq_append_decode_attention(kvq_cache* c, int32_t layer, const void* k_new, const void* v_new,
                                const void* q, const int32_t* seq_lens, const int32_t* page_table,
                                int32_t batch, float softmax_scale, void* out, void* stream) {
  if (c && batch > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)))
    return KVQ_EINVAL;
  return decode_common(c, layer, k_new, v_new, q, seq_lens, page_table, batch, softmax_scale, out,
                       stream);
}

int kvq_prefill_attention(kvq_cache* c, int32_t layer, const void* q, const int32_t* cu_q,
                          const int32_t* seq_lens, const int32_t* page_table, int32_t batch,
                          int32_t total_q, float softmax_scale, void* out, void* stream) {
  if (!c) return KVQ_EINVAL;
  if (layer < 0 || layer >= c->d.num_layers) return KVQ_EINVAL;
  if (batch < 0 || batch > c->d.max_batch || total_q < 0) return KVQ_EINVAL;
  if (!(softmax_scale >= 0.0f) || isinf(softmax_scale)) return KVQ_EINVAL;
  if (batch == 0 || total_q == 0) return KVQ_OK;
  if (!q || !cu_q || !seq_lens || !page_table || !out) return KVQ_EINVAL;
  if (!aligned16(q) || !aligned16(out)) return KVQ_EINVAL;
  kvq::PrefillParams p;
  const size_t layer_bytes = pool_bytes_of(&c->d) / c->d.num_layers;
  p.pool_layer = c->pool + static_cast<size_t>(layer) * layer_bytes;
  p.q = static_cast<const __half*>(q);
  p.cu_q = cu_q;
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.out = static_cast<__half*>(out);
  p.status = c->status;
  p.batch = batch;
  p.num_kv_heads = c->d.num_kv_heads;
  p.group = c->d.num_q_heads / c->d.num_kv_heads;
  p.num_pages = c->d.num_pages;
  p.page_size = c->d.page_size;
  p.page_shift = __builtin_ctz(static_cast<unsigned>(c->d.page_size));
  p.max_pages_per_seq = c->d.max_pages_per_seq;
  p.hadamard_block = c->d.hadamard_block;
  const double sm = softmax_scale == 0.0f ? 1.0 / sqrt(static_cast<double>(c->d.head_dim))
                                          : static_cast<double>(softmax_scale);
  p.q_scale = static_cast<float>(sm * 1.4426950408889634);  // log2(e)
  p.cb = c->cb;
  p.fp4 = c->d.kv_format == KVQ_FORMAT_NVFP4;
  const int rc = kvq::launch_prefill_tc(p, total_q, static_cast<cudaStream_t>(stream));
  if (rc == -1) return KVQ_EUNSUPPORTED;
  return rc == 0 ? KVQ_OK : KVQ_ECUDA;
}

void* kvq_pool_ptr(const kvq_cache* c) { return c ? c->pool : nullptr; }

int kvq_get_device_status(kvq_cache* c, int32_t* status, void* stream) {
  if (!c || !status) return KVQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, c->status, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return KVQ_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ECUDA;
  if (cudaMemsetAsync(c->status, 0, sizeof v, s) != cudaSuccess) return KVQ_ECUDA;
  *status = v;
  return KVQ_OK;
}

int kvq_free(kvq_cache* c) {
  if (!c) return KVQ_OK;
  int rc = KVQ_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) rc = KVQ_ECUDA;
  if (c->own_pool && cudaFree(c->pool) != cudaSuccess) rc = KVQ_ECUDA;
  if (cudaFree(c->scratch) != cudaSuccess) rc = KVQ_ECUDA;
  delete c;
  return rc;
}

}  // extern "C"

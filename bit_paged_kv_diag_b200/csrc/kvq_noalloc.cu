// kvq_noalloc.cu -- decode attention for callers that cannot allocate device memory.
//
// kvq_decode_attention needs a kvq_cache handle, and creating one calls cudaMalloc for the
// split scratch.  Some callers cannot do that: an inference runtime that has reserved all
// of device memory for its own pool and forbids stray allocations, a plugin whose host
// framework owns every device allocation, or a latency-critical path where cudaMalloc's
// implicit device synchronisation is not acceptable.  kvq_decode_attention_noalloc runs the
// same decode kernel with its scratch (status word, per-unit arrival counters, per-CTA
// partials) in one file-scope __device__ array of fixed size, so it allocates nothing.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/kvq.h"
#include "kvq_internal.h"

namespace {

// Static scratch: [status word, padded to 256 B][arrival counters][partial records].
constexpr int kNoAllocMaxUnits = 4096;    // batch * num_kv_heads
constexpr int kNoAllocMaxRecords = 4096;  // (batch * num_kv_heads + grid CTAs) * G
constexpr size_t kNoAllocCounterBytes = kNoAllocMaxUnits * sizeof(int32_t);
constexpr size_t kNoAllocBytes =
    256 + kNoAllocCounterBytes + static_cast<size_t>(kNoAllocMaxRecords) * kvq::kDecodeWarps *
                                     kvq::kPartStride * sizeof(float);

// Every GPU that loads the library holds this array (about 8.7 MB) until exit.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
unsigned char* g_scratch_addr[kMaxDevices];  // device address of the array, per device
int g_num_sms[kMaxDevices];

// Once per device, with that device current: the array's device address (its name in
// host code is only a host-side stand-in) and zeroed counters.
int setup_device(int dev, unsigned char** scratch, int* num_sms) {
  if (dev < 0 || dev >= kMaxDevices) return KVQ_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return KVQ_ECUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return KVQ_ECUDA;
    if (cudaMemset(addr, 0, 256 + kNoAllocCounterBytes) != cudaSuccess) return KVQ_ECUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return KVQ_ECUDA;
    g_num_sms[dev] = sms;
    g_scratch_addr[dev] = static_cast<unsigned char*>(addr);
  }
  *scratch = g_scratch_addr[dev];
  *num_sms = g_num_sms[dev];
  return KVQ_OK;
}

bool noalloc_desc_ok(const kvq_desc* d) {
  if (!d || d->num_layers < 1 || d->num_kv_heads < 1 || d->num_q_heads < 1 ||
      d->num_pages < 1 || d->max_batch < 1 || d->max_pages_per_seq < 1)
    return false;
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
  const long long tiles_per_seq = (static_cast<long long>(d->max_pages_per_seq) * S + 31) / 32;
  if (static_cast<long long>(d->max_batch) * d->num_kv_heads * tiles_per_seq >= (1LL << 30))
    return false;
  return true;
}

}  // namespace

extern "C" {

int kvq_decode_attention_noalloc(const kvq_desc* d, const void* pool, int32_t layer,
                                 const void* q, const int32_t* seq_lens,
                                 const int32_t* page_table, int32_t batch, float softmax_scale,
                                 void* out, void* stream) {
  if (!noalloc_desc_ok(d)) return d ? KVQ_EUNSUPPORTED : KVQ_EINVAL;
  if (layer < 0 || layer >= d->num_layers) return KVQ_EINVAL;
  if (batch < 0 || batch > d->max_batch) return KVQ_EINVAL;
  if (!(softmax_scale >= 0.0f) || isinf(softmax_scale)) return KVQ_EINVAL;
  if (batch == 0) return KVQ_OK;
  if (!pool || !q || !seq_lens || !page_table || !out) return KVQ_EINVAL;
  const uintptr_t a16 = 15u;
  if ((reinterpret_cast<uintptr_t>(pool) | reinterpret_cast<uintptr_t>(q) |
       reinterpret_cast<uintptr_t>(out)) & a16)
    return KVQ_EINVAL;
  const int g = d->num_q_heads / d->num_kv_heads;
  const long long units = static_cast<long long>(batch) * d->num_kv_heads;
  if (units > kNoAllocMaxUnits) return KVQ_EUNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ECUDA;
  unsigned char* scratch = nullptr;
  int num_sms = 0;
  const int rc = setup_device(dev, &scratch, &num_sms);
  if (rc != KVQ_OK) return rc;

  kvq::DecodeLaunch L;
  const int fp4 = d->kv_format == KVQ_FORMAT_NVFP4;
  if (kvq::plan_decode(g, d->page_size, batch, num_sms, fp4, &L) != 0) return KVQ_ECUDA;
  if ((units + L.grid) * g > kNoAllocMaxRecords) return KVQ_EUNSUPPORTED;

  kvq::DecodeParams p;
  const size_t layer_bytes = static_cast<size_t>(d->num_pages) * d->num_kv_heads *
                             d->page_size * (d->head_dim + (fp4 ? d->head_dim / 8 : 4));
  p.pool_layer = static_cast<const uint8_t*>(pool) + static_cast<size_t>(layer) * layer_bytes;
  p.q = static_cast<const __half*>(q);
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.out = static_cast<__half*>(out);
  p.status = reinterpret_cast<int32_t*>(scratch);
  p.counters = reinterpret_cast<int32_t*>(scratch + 256);
  p.part = reinterpret_cast<float*>(scratch + 256 + kNoAllocCounterBytes);
  p.batch = batch;
  p.num_kv_heads = d->num_kv_heads;
  p.group = g;
  p.num_pages = d->num_pages;
  p.page_size = d->page_size;
  p.page_shift = __builtin_ctz(static_cast<unsigned>(d->page_size));
  p.max_pages_per_seq = d->max_pages_per_seq;
  p.hadamard_block = d->hadamard_block;
  const double sm = softmax_scale == 0.0f ? 1.0 / sqrt(static_cast<double>(d->head_dim))
                                          : static_cast<double>(softmax_scale);
  p.q_scale = static_cast<float>(sm * 1.4426950408889634);  // log2(e)
  p.cb = static_cast<float>(1.0 / sqrt(static_cast<double>(d->hadamard_block)));
  p.total_ctas = L.grid;
  p.k_new = nullptr;
  p.v_new = nullptr;
  p.fp4 = fp4;
  const int lrc = kvq::launch_decode(p, L, static_cast<cudaStream_t>(stream));
  if (lrc == -1) return KVQ_EUNSUPPORTED;
  return lrc == 0 ? KVQ_OK : KVQ_ECUDA;
}

}  // extern "C"

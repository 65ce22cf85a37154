// kvq_noalloc.cu -- decode attention for callers that cannot allocate device memory.
//
// kvq_decode_attention needs a kvq_cache handle, and creating one calls cudaMalloc for the
// split scratch.  Some callers cannot do that: an inference runtime that has reserved all
// of device memory for its own pool and forbids stray allocations, a plugin whose host
// framework owns every device allocation, or a latency-critical path where cudaMalloc's
// implicit device synchronisation is not acceptable.  kvq_decode_attention_noalloc runs the
// same decode kernel with its scratch (per-unit arrival counters, per-CTA partials, and a
// status word for callers that pass none) in one file-scope __device__ array of fixed size,
// so it allocates nothing.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/kvq.h"
#include "kvq_internal.h"

namespace {

// Static scratch: [status word, padded to 256 B][arrival counters][partial records].
// The records bound the call: (batch * num_kv_heads + grid CTAs) * G <= kNoAllocMaxRecords.
// That bound also keeps batch * num_kv_heads below kNoAllocMaxUnits, the size of the
// counter array (one counter per (sequence, KV head) unit).
constexpr int kNoAllocMaxUnits = 4096;
constexpr int kNoAllocMaxRecords = 4096;
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

// Launch shapes already planned, so a call after the first for a given shape makes no
// attribute or occupancy queries.  Keyed by device, G, page size, format and the batch
// rounded up to a power of two (the plan's shared memory holds per-sequence arrays).
struct PlanEntry {
  int dev, g, page_size, fp4, batch_cap;
  kvq::DecodeLaunch launch;
};
constexpr int kMaxPlans = 256;
PlanEntry g_plans[kMaxPlans];
int g_num_plans = 0;

// The array's device address on the current device (its name in host code is only a
// host-side stand-in), looked up on every call: the lookup is a host-side query that
// allocates nothing, and it stays right if the context was reset since the last call.
// The first time an address is seen on a device, the counters are zeroed (synchronising
// the device); a module loaded anew after a reset starts zeroed as well.
int scratch_for(int dev, unsigned char** scratch, int* num_sms) {
  if (dev < 0 || dev >= kMaxDevices) return KVQ_EUNSUPPORTED;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return KVQ_ECUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_addr[dev] != addr) {
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

// Returns 0, -1 (shape the decode kernel does not implement) or -2 (CUDA error).
int plan_for(int dev, int g, int page_size, int fp4, int batch, int num_sms, kvq::DecodeLaunch* L) {
  int cap = 16;
  while (cap < batch) cap *= 2;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  for (int i = 0; i < g_num_plans; i++) {
    const PlanEntry& e = g_plans[i];
    if (e.dev == dev && e.g == g && e.page_size == page_size && e.fp4 == fp4 && e.batch_cap == cap) {
      *L = e.launch;
      return 0;
    }
  }
  const int rc = kvq::plan_decode(g, page_size, cap, num_sms, fp4, L);
  if (rc != 0) return rc;
  if (g_num_plans < kMaxPlans) g_plans[g_num_plans++] = PlanEntry{dev, g, page_size, fp4, cap, *L};
  return 0;
}

}  // namespace

extern "C" {

int kvq_decode_attention_noalloc(const kvq_desc* d, const void* pool, size_t pool_bytes,
                                 int32_t layer, const void* q, const int32_t* seq_lens,
                                 const int32_t* page_table, int32_t batch, float softmax_scale,
                                 void* out, int32_t* dev_status, void* stream) {
  int why = KVQ_OK;
  if (!kvq::desc_valid(d, &why)) return why;
  if (layer < 0 || layer >= d->num_layers) return KVQ_EINVAL;
  if (batch < 0 || batch > d->max_batch) return KVQ_EINVAL;
  if (!(softmax_scale >= 0.0f) || isinf(softmax_scale)) return KVQ_EINVAL;
  if (batch == 0) return KVQ_OK;
  if (!pool || !q || !seq_lens || !page_table || !out) return KVQ_EINVAL;
  const size_t layer_bytes = kvq::desc_layer_bytes(d);
  if (pool_bytes < static_cast<size_t>(d->num_layers) * layer_bytes) return KVQ_EINVAL;
  const uintptr_t a16 = 15u;
  if ((reinterpret_cast<uintptr_t>(pool) | reinterpret_cast<uintptr_t>(q) |
       reinterpret_cast<uintptr_t>(out)) & a16)
    return KVQ_EINVAL;
  if (reinterpret_cast<uintptr_t>(dev_status) & 3u) return KVQ_EINVAL;
  const int g = d->num_q_heads / d->num_kv_heads;
  const long long units = static_cast<long long>(batch) * d->num_kv_heads;
  if (units > kNoAllocMaxUnits) return KVQ_EUNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ECUDA;
  unsigned char* scratch = nullptr;
  int num_sms = 0;
  const int rc = scratch_for(dev, &scratch, &num_sms);
  if (rc != KVQ_OK) return rc;

  kvq::DecodeLaunch L;
  const int fp4 = d->kv_format == KVQ_FORMAT_NVFP4;
  const int prc = plan_for(dev, g, d->page_size, fp4, batch, num_sms, &L);
  if (prc == -1) return KVQ_EUNSUPPORTED;
  if (prc != 0) return KVQ_ECUDA;
  if ((units + L.grid) * g > kNoAllocMaxRecords) return KVQ_EUNSUPPORTED;

  kvq::DecodeParams p;
  p.pool_layer = static_cast<const uint8_t*>(pool) + static_cast<size_t>(layer) * layer_bytes;
  p.q = static_cast<const __half*>(q);
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.out = static_cast<__half*>(out);
  p.status = dev_status ? dev_status : reinterpret_cast<int32_t*>(scratch);
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

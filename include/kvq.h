/*
 * kvq.h -- C ABI of libkvq.so: rotated-INT4 paged KV cache on NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources cited by page title and section):
 *
 *   [P1] "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化" (youngju.dev)
 *   [P2] "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving"
 *        (gist.science)
 *   [P3] "BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号" (sns.style): the NVFP4
 *        cache format, kv_format = KVQ_FORMAT_NVFP4 below
 *
 *   * Every new K/V row (fp16, head_dim = 128 channels) is rotated by an orthonormal
 *     block-diagonal Hadamard transform (blocks of b = 32, 64 or 128 channels) [P1,
 *     "回転のトリック — ブロック対角アダマール"], quantised token-wise to symmetric INT4
 *     with one fp16 scale per token per KV head [P1, "素朴なINT4はなぜ崩れるのか"], and
 *     appended into fixed-size pages addressed through a page table, without touching
 *     past tokens [P1, "システムこそが設計である — 融合カーネル"].
 *   * Paged GQA decode attention reads that cache: q is rotated with the same transform,
 *     pages are dequantised in-kernel, softmax is computed online, and the output is
 *     rotated back (the orthonormal Sylvester matrix is its own inverse) [P1,
 *     "KVキャッシュこそが本当のボトルネックである理由": paged layout, fused attention].
 *
 * Readings of what the pages leave open (the CPU oracle takes the same readings):
 *   rotation   fp32 butterfly, stages h = 1, 2, ..., b/2, then one multiply by the fp32
 *              value nearest 1/sqrt(b); natural (Sylvester) order;
 *   scale      s = fp16_rn(max_d |y_d| / 7) over all 128 channels, saturated at 65504;
 *   codes      clamp(round_half_even(y_d / s), -8, 7), dividing by the stored fp16 s;
 *              all codes 0 when s == 0;
 *   packing    two codes per byte, low nibble = even channel, 4-bit two's complement;
 *   GQA        query head hq reads KV head hq / (num_q_heads / num_kv_heads);
 *   softmax    scale 1/sqrt(head_dim) unless given; an empty sequence outputs zeros.
 *
 * NVFP4 format (kv_format = KVQ_FORMAT_NVFP4) [P3, "背景と概要", "深掘り分析": a 4-bit
 * microscaling format with E4M3 block scales; the pages give no formulas, the readings]:
 *   the same rotation; then per block of 16 channels an E4M3 scale s = the fp32 value
 *   max |y| / 6 rounded to nearest even and saturated at 448; codes = E2M1 (sign, 2
 *   exponent bits, 1 mantissa bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6) nearest to y * (1/s)
 *   (fp32 reciprocal and product), ties to the even code, saturated at 6, the sign kept;
 *   all codes 0 when s == 0; no per-tensor scale.  Packing as for INT4.
 *
 * Pool layout (device memory, bytes; one pool holds every layer):
 *   block(layer, page, kv_head) starts at
 *       ((layer * num_pages + page) * num_kv_heads + kv_head) * page_size * R
 *   with R = 132 (INT4) or 144 (NVFP4), and holds, for the page_size token slots:
 *       [K codes  page_size x 64 B][V codes  page_size x 64 B]
 *       [K scales page_size x fp16][V scales page_size x fp16]           (INT4)
 *       [K scales page_size x 8 E4M3][V scales page_size x 8 E4M3]       (NVFP4: block j
 *                                                          of a row = channels 16j..16j+15)
 *   Token at position pos of sequence b lives in page page_table[b][pos / page_size],
 *   slot pos % page_size.  The page table is shared by all layers.
 *
 * Conventions for every call:
 *   * Return value: KVQ_OK (0) or a negative status below.  Argument errors that the
 *     host can see are returned before anything is launched.
 *   * Calls that launch work are asynchronous and ordered on the given stream (a
 *     cudaStream_t passed as void*; NULL = the legacy default stream).  They never
 *     synchronise the host.  Asynchronous CUDA errors surface at the caller's next
 *     synchronisation.
 *   * A bad page id or an out-of-range position met on the device (a page-table entry
 *     outside [0, num_pages), a position beyond max_pages_per_seq * page_size) is never
 *     a trap: the kernel skips or redirects the access and ORs a code into the handle's
 *     device status word, read with kvq_get_device_status().
 *   * No C++ exception crosses this boundary.  No call changes seq_lens or the page
 *     table; the caller advances seq_lens by the number of appended tokens.
 *   * Ownership: the caller owns q, k, v, out, seq_lens, page_table and (optionally) the
 *     pool; the library owns the handle, its split-KV scratch, its status word and the
 *     pool when it allocated it.  One handle must not be used from two streams at once
 *     (decode calls share the handle's scratch).
 *   * Launch overlap: every kernel of this library uses programmatic dependent launch.  Each lets the next
 *     kernel on the stream start at its own entry, and waits for the previous kernel to
 *     complete before it touches the pool, q, out or the handle's scratch.  Before that
 *     wait, decode already reads seq_lens and page_table, append reads k, v,
 *     cu_new_tokens, seq_lens and page_table, and the fused append + decode reads k_new,
 *     v_new, seq_lens and page_table, and prefill attention reads cu_q, seq_lens and
 *     page_table.  These arrays must therefore be complete
 *     when the previous kernel on the stream lets its dependents start.  Kernels that do
 *     not use programmatic launch (PyTorch's, cuBLAS's, copies) only do so by completing,
 *     and this library's own kernels never write these arrays.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define KVQ_OK 0
#define KVQ_EINVAL (-1)        /* a null pointer, a negative size, a misaligned buffer  */
#define KVQ_EUNSUPPORTED (-2)  /* a shape outside what the kernels implement            */
#define KVQ_ENOPAGES (-3)      /* the pool or a sequence's page budget is too small      */
#define KVQ_ECUDA (-4)         /* a CUDA runtime call failed (allocation, launch, copy)  */

/* Bits of the device status word (kvq_get_device_status). */
#define KVQ_DEV_BAD_PAGE 1     /* a page-table entry outside [0, num_pages)              */
#define KVQ_DEV_BAD_POS 2      /* a position or length beyond the sequence's page budget */
#define KVQ_DEV_TIMEOUT 4      /* a bounded wait in a kernel gave up (never expected)    */

typedef struct kvq_cache kvq_cache; /* opaque, library-owned handle */

/* Cache geometry; all values are host integers.
 *   num_layers         layers sharing one pool and one page table            (>= 1)
 *   num_kv_heads       Hkv                                                    (>= 1)
 *   num_q_heads        Hq, a multiple of Hkv; G = Hq / Hkv must be 1, 2, 4 or 8
 *   head_dim           D; only 128 is implemented
 *   hadamard_block     b: 32, 64 or 128; or 1 for plain token-wise INT4 without the
 *                      rotation (the transform with b = 1 is the identity and c_b = 1)
 *   page_size          S tokens per page: 16, 32, 64, 128 or 256
 *   num_pages          pages per layer in the pool                            (>= 1)
 *   max_batch          largest batch any call will pass                (1 .. 4096)
 *   max_pages_per_seq  row length of the page table                          (>= 1)
 *   kv_format          KVQ_FORMAT_INT4 (0) or KVQ_FORMAT_NVFP4 (1); every call supports
 *                      both formats */
#define KVQ_FORMAT_INT4 0
#define KVQ_FORMAT_NVFP4 1
typedef struct {
  int32_t num_layers;
  int32_t num_kv_heads;
  int32_t num_q_heads;
  int32_t head_dim;
  int32_t hadamard_block;
  int32_t page_size;
  int32_t num_pages;
  int32_t max_batch;
  int32_t max_pages_per_seq;
  int32_t kv_format;
} kvq_desc;

/* Bytes of the pool a descriptor needs:
 * num_layers * num_pages * num_kv_heads * page_size * R (R = 132 INT4, 144 NVFP4).
 * Returns 0 for an invalid descriptor.  Host only. */
KVQ_API size_t kvq_pool_bytes(const kvq_desc* d);

/* Deterministic page assignment (host only; no CUDA call).  Walks page_order (host
 * [num_pages], a permutation of 0..num_pages-1) or, when page_order is NULL, the pages
 * 0..num_pages-1, and gives sequence b = 0, 1, ..., batch-1 in turn the next
 * ceil(capacity_tokens[b] / page_size) pages.
 *   capacity_tokens  host [batch], tokens each sequence must be able to hold (>= 0)
 *   page_table       host out [batch][max_pages_per_seq]; unused entries are -1
 * Returns KVQ_OK, KVQ_EINVAL, KVQ_EUNSUPPORTED (descriptor), or KVQ_ENOPAGES when a
 * sequence needs more than max_pages_per_seq pages or the pool runs out.  The page
 * table is then left partially written. */
KVQ_API int kvq_assign_pages(const kvq_desc* d, int32_t batch, const int32_t* capacity_tokens,
                     const int32_t* page_order, int32_t* page_table);

/* Create a cache handle, the split-KV scratch and (optionally) the pool, and assign
 * pages with kvq_assign_pages: the pages' fixed-size KV blocks addressed through a page
 * table ("KVキャッシュを4ビットへ", section "KVキャッシュこそが本当のボトルネックである理由").
 *   dev_pool    device buffer of >= kvq_pool_bytes(d) bytes, 16-byte aligned, owned by
 *               the caller; NULL = the library allocates (cudaMalloc) and owns the pool
 *   pool_bytes  size of dev_pool (ignored when dev_pool is NULL)
 *   batch, capacity_tokens, page_order, page_table: as kvq_assign_pages; batch may be
 *               0 (then no table is written) and must not exceed max_batch
 *   out         receives the handle
 * Uses the current CUDA device.  Blocks the host (allocation).  Returns KVQ_OK or a
 * negative status; on failure nothing is left allocated and *out is NULL. */
KVQ_API int kvq_alloc_pages(const kvq_desc* d, void* dev_pool, size_t pool_bytes, int32_t batch,
                    const int32_t* capacity_tokens, const int32_t* page_order,
                    int32_t* page_table, kvq_cache** out);

/* Fused block-diagonal Hadamard rotation + token-wise INT4 quantisation + paged append
 * for one layer [P1, "システムこそが設計である — 融合カーネル"]; NVFP4 rows instead
 * for a cache with kv_format = KVQ_FORMAT_NVFP4.  One kernel launch.
 *   layer             0 .. num_layers-1
 *   k, v              device fp16 [total_new_tokens][num_kv_heads][128], token-major,
 *                     32-byte aligned (rows are read with 256-bit loads)
 *   cu_new_tokens     device int32 [batch+1], cu[0] = 0, non-decreasing,
 *                     cu[batch] = total_new_tokens; sequence b appends tokens
 *                     cu[b] .. cu[b+1]-1 of k/v
 *   seq_lens          device int32 [batch], lengths BEFORE this append
 *   page_table        device int32 [batch][max_pages_per_seq]
 *   batch             0 .. max_batch;  total_new_tokens >= 0 (0 launches nothing)
 * Token i of sequence b is written at position seq_lens[b] + i.  Nothing else in the
 * pool is written.  Returns KVQ_OK or a negative status (before any launch). */
KVQ_API int kvq_rotate_quant_append(kvq_cache* c, int32_t layer, const void* k, const void* v,
                            const int32_t* cu_new_tokens, const int32_t* seq_lens,
                            const int32_t* page_table, int32_t batch,
                            int32_t total_new_tokens, void* stream);

/* Paged GQA decode attention over the cache (INT4 or NVFP4) of one layer: one query
 * token per sequence.  The pages' fused attention over the paged, quantised cache, q
 * rotated with the cache's transform and the output rotated back ("KVキャッシュを4ビットへ",
 * sections "KVキャッシュこそが本当のボトルネックである理由" and "回転のトリック —
 * ブロック対角アダマール").  One kernel launch: a split-KV pass whose last-arriving CTA per (sequence,
 * KV head) merges the splits and applies the inverse rotation.
 *   q              device fp16 [batch][num_q_heads][128], 16-byte aligned
 *   seq_lens       device int32 [batch], lengths AFTER any append (tokens to attend)
 *   page_table     device int32 [batch][max_pages_per_seq]
 *   batch          0 .. max_batch
 *   softmax_scale  multiplier of q.k; 0 means 1/sqrt(128)
 *   out            device fp16 [batch][num_q_heads][128], 16-byte aligned; rows of
 *                  empty sequences are zeros
 * Uses the handle's scratch: calls on one handle must be ordered (one stream).
 * Returns KVQ_OK or a negative status (before any launch). */
KVQ_API int kvq_decode_attention(kvq_cache* c, int32_t layer, const void* q, const int32_t* seq_lens,
                         const int32_t* page_table, int32_t batch, float softmax_scale,
                         void* out, void* stream);

/* Append one token per sequence and decode over it, in one launch: the fused form of
 * kvq_rotate_quant_append (one new token per sequence, cu_new_tokens = 0, 1, ..., batch)
 * followed by kvq_decode_attention.  It follows the pages' fused kernel that rotates,
 * quantises and appends as the token is produced ("KVキャッシュを4ビットへ", section
 * "システムこそが設計である — 融合カーネル"), and also saves the second launch per
 * layer in a decode step.  The pool receives exactly the bytes the separate append would
 * write.
 *   k_new, v_new   device fp16 [batch][num_kv_heads][128], 16-byte aligned: the new
 *                  token's K and V rows
 *   seq_lens       device int32 [batch], lengths BEFORE the append: the new token goes to
 *                  position seq_lens[b] and the decode attends seq_lens[b] + 1 tokens
 *   q, page_table, batch, softmax_scale, out, stream: as for kvq_decode_attention
 * A position beyond the sequence's page budget or a bad page id is flagged in the status
 * word (KVQ_DEV_BAD_POS / KVQ_DEV_BAD_PAGE) and that row is not stored.
 * Returns KVQ_OK or a negative status (before any launch). */
KVQ_API int kvq_append_decode_attention(kvq_cache* c, int32_t layer, const void* k_new,
                                        const void* v_new, const void* q,
                                        const int32_t* seq_lens, const int32_t* page_table,
                                        int32_t batch, float softmax_scale, void* out,
                                        void* stream);

/* Causal chunked-prefill attention over the cache (INT4 or NVFP4) of one layer: many
 * query tokens per sequence.  A chunk of C_b = cu_q[b+1] - cu_q[b] prompt tokens of sequence b, already
 * appended (kvq_rotate_quant_append), attends the cache causally: query i of the chunk,
 * at position seq_lens[b] - C_b + i, attends positions 0 .. seq_lens[b] - C_b + i.  The
 * pages' attention over the paged cache ("KVキャッシュを4ビットへ", section
 * "KVキャッシュこそが本当のボトルネックである理由") for the many-query case a serving
 * engine runs on the same cache; decode is the case C_b = 1.  Runs on the 5th-generation
 * tensor cores (tcgen05 MMAs, S and O in tensor memory, one CTA of 128 query rows per SM,
 * 512 tensor-memory columns) for both cache formats.
 *   q              device fp16 [total_q][num_q_heads][128], the chunks concatenated in
 *                  order of b, 16-byte aligned
 *   cu_q           device int32 [batch+1], chunk offsets into q (cu_q[0] = 0)
 *   seq_lens       device int32 [batch], tokens cached, the chunk included (C_b <=
 *                  seq_lens[b] <= max_pages_per_seq * page_size)
 *   page_table     device int32 [batch][max_pages_per_seq]
 *   total_q        host int32, cu_q[batch] (sizes the launch)
 *   softmax_scale  multiplier of q.k; 0 means 1/sqrt(128)
 *   out            device fp16 [total_q][num_q_heads][128], 16-byte aligned
 * A chunk longer than its sequence, or a length beyond the page budget, is flagged
 * (KVQ_DEV_BAD_POS) and its rows are not written.  Uses no scratch; calls on one handle
 * may run on any stream ordering the caller chooses.  Returns KVQ_OK or a negative status
 * (before any launch). */
KVQ_API int kvq_prefill_attention(kvq_cache* c, int32_t layer, const void* q,
                                  const int32_t* cu_q, const int32_t* seq_lens,
                                  const int32_t* page_table, int32_t batch, int32_t total_q,
                                  float softmax_scale, void* out, void* stream);

/* Decode attention that allocates nothing.  The pages have no counterpart of this call;
 * it exists for callers that cannot call cudaMalloc: an inference runtime that has
 * reserved all of device memory for its own pool and forbids stray allocations, a plugin
 * whose host framework owns every device allocation, or a latency-critical path where
 * cudaMalloc's implicit device synchronisation is not acceptable.  Those callers cannot
 * create a kvq_cache (kvq_alloc_pages allocates the split scratch), so this call takes the
 * geometry and the pool directly and keeps its scratch in one fixed-size device array
 * inside the library (about 8.7 MB, held by every GPU that loads the library until exit).
 *   d              cache geometry (as for kvq_alloc_pages); only read
 *   pool           device pool, 16-byte aligned, laid out as kvq_rotate_quant_append
 *                  writes it (caller-owned)
 *   pool_bytes     size of pool; less than kvq_pool_bytes(d) is KVQ_EINVAL
 *   dev_status     device int32, 4-byte aligned, caller-owned: the kernel ORs KVQ_DEV_*
 *                  bits into it (the caller reads and clears it); NULL = the bits go to a
 *                  word inside the library's array that is never read
 *   layer, q, seq_lens, page_table, batch, softmax_scale, out, stream: as for
 *                  kvq_decode_attention
 * Limits of the fixed scratch: (batch * num_kv_heads + C) * G <= 4096, C = the kernel's
 * grid (up to 3 CTAs per SM); a larger call returns KVQ_EUNSUPPORTED before anything is
 * launched.
 * The first call on a device (and the first after a context reset) sets the array up:
 * it zeroes the arrival counters, which synchronises the device; make that first call
 * before any stream capture.  Later calls look up the array's address (a host-side query)
 * and reuse the launch shape planned for their (G, page size, format, batch) class.
 * Every call shares the array: calls that overlap on the GPU (two streams, or two
 * processes' contexts on one device) race on it and must be ordered by the caller.  A
 * call whose bounded wait gave up (KVQ_DEV_TIMEOUT in dev_status) has undefined outputs,
 * but every CTA of it still arrives on the counters it uses, so the counters are back at
 * zero when it ends and later calls are unaffected.  Returns KVQ_OK or a negative status. */
KVQ_API int kvq_decode_attention_noalloc(const kvq_desc* d, const void* pool, size_t pool_bytes,
                                         int32_t layer, const void* q, const int32_t* seq_lens,
                                         const int32_t* page_table, int32_t batch,
                                         float softmax_scale, void* out, int32_t* dev_status,
                                         void* stream);

/* Device address of the pool (the caller's buffer, or the library's). NULL for NULL. */
KVQ_API void* kvq_pool_ptr(const kvq_cache* c);

/* Read and clear the handle's device status word (KVQ_DEV_* bits).  Synchronises the
 * given stream.  Returns KVQ_OK or KVQ_ECUDA / KVQ_EINVAL. */
KVQ_API int kvq_get_device_status(kvq_cache* c, int32_t* status, void* stream);

/* Free library-owned memory (the handle, scratch, status word, and the pool if the
 * library allocated it): the release of the paged cache that kvq_alloc_pages created
 * ("KVキャッシュを4ビットへ", section "KVキャッシュこそが本当のボトルネックである理由").  Synchronises the device first.  NULL is a no-op.  Returns
 * KVQ_OK, or KVQ_ECUDA if an earlier asynchronous error is found. */
KVQ_API int kvq_free(kvq_cache* c);

/* Short static description of a status code. */
KVQ_API const char* kvq_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */

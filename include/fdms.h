/*
 * fdms.h - C ABI of the compact-KV decode-attention library (sm_100a).
 *
 * The method: DMS learns, per attention head, which tokens' KV slots to drop;
 * FastDMS keeps only the survivors, in a compact store that physically
 * reclaims the dropped slots, next to a staging area, and decodes over that
 * store in BF16 or FP8 ("FastDMS: 6.4X KV-cache compression running faster
 * than vLLM BF16/FP8", aiwitness.kr/community/1t3vlrx: the paragraphs on DMS
 * per-head eviction and on the compact store, and the KV-memory table with its
 * BF16 / FP8 columns and "KV/stage memory = cache, or cache + staging").
 *
 * This library holds that cache on one GPU and runs the three steps of a decode
 * layer on it:
 *   fdms_append_evict  - append new tokens, apply the keep decision of tokens
 *                        that leave the recent window, compact survivors;
 *   fdms_decode_attn   - single-token attention of every query head over the
 *                        survivors of its kv head (split over the GPU, then
 *                        merged: through distributed shared memory inside a
 *                        cluster of CTAs per head for calls with few heads, by
 *                        the last split warp of each head to finish otherwise;
 *                        one kernel either way);
 *   fdms_cache_stats   - counters, including compact vs dense-equivalent bytes
 *                        (the quantity of the pages' KV-memory table).
 *
 * Semantics (the pages give none in detail; these are the readings used):
 *   - Per (layer, seq, kv head) the tokens have positions 0..n-1. Token j is
 *     visible to decode iff j >= n - W (recent window) or keep[j] = 1.
 *   - A token's keep bit is applied when it is resolved: resolution runs after
 *     an append that leaves at least P out-of-window tokens unresolved, and then
 *     resolves all of them (P = 1: each token as it leaves the window). Kept
 *     tokens are appended, in position order, to the head's compact store;
 *     the others are dropped and their memory is never used.
 *   - Unresolved tokens (at most W + P - 1 per head) live in a per-head ring:
 *     the staging area.
 *   - Query head i reads kv head floor(i / G), G = num_q_heads / num_kv_heads.
 *   - Decode runs after the step's token is appended (it attends to itself).
 *   - FP8 E4M3 cache: each (layer, seq, kv head) gets one fp32 scale for K and
 *     one for V at its first append (max(amax, 2^-126) / 448 over that call's
 *     values, or the caller's); a value is stored as
 *     e4m3_rne_satfinite(fp32(x) / scale). Each 64-slot store block carries its
 *     own scale pair, which decode applies per block.
 *
 * Memory and ownership: the cache owns all device memory it allocates at
 * fdms_cache_create (pool, tables, ring, decode workspace) and frees it at
 * fdms_cache_destroy. The caller owns every buffer passed in (inputs, outputs,
 * streams) and keeps them alive until the work queued on the stream is done.
 * No call allocates device memory after creation.
 *
 * Ordering and threads: queue the calls on one cache in program order on one
 * stream, or order streams with events. Consecutive kernels on a stream overlap
 * through programmatic dependent launch: a kernel may start while the one
 * before it finishes, and reads what that kernel writes only after its
 * dependency wait. Before the wait a kernel reads only cache state that a
 * kernel queued earlier has certainly finished writing: the cache keeps a
 * host-side log of the kernels it queued, and every kernel that starts has
 * seen each kernel before the last "wait-first" kernel (one whose every CTA
 * waits before it lets its dependents start) complete. Kernels of other code
 * queued between the library's calls keep that true as long as none of them
 * lets its dependents start before its own dependency wait (kernels launched
 * without programmatic dependent launch never do). Because of that host-side
 * state, calls on one cache must not run concurrently from several host
 * threads; different caches are independent.
 *
 * Stream capture: the calls may be captured into a CUDA graph (the host-side
 * record of the cache is updated when a call is captured). Each launch of such
 * a graph then stands for the captured calls in their place in the cache's
 * call order: launch it exactly once, where the captured calls would have run.
 * A graph launched several times would plan its decode calls from records of
 * the first time (which snapshot copy to read, how many tokens were appended
 * since), which later launches no longer match.
 *
 * Errors: every call validates its arguments on the host and returns a status
 * before queuing any work. Calls that queue kernels are asynchronous; errors
 * found by the device (pool exhausted, sequence too long) are latched into a
 * sticky word with the first error code and the affected head is left
 * unchanged; fdms_cache_stats reports the word. Device code never traps or
 * waits without a bound (the barriers of one CTA or one cluster aside, which
 * every thread of it reaches): a decode wait on its tile copies gives up after
 * 2 s, latches FDMS_ERR_DEVICE and the kernel still finishes. For tests of that
 * path, a cache created while the environment variable FDMS_TEST_STALL_COPIES
 * is set (and not "0") has every decode tile stage expect 16 bytes more than
 * its copies bring, so that its decode waits run out.
 *
 * Layouts: all tensors are dense, row-major, in the order written; "bf16" is
 * the IEEE binary32 upper half. Device pointers must be 16-byte aligned.
 * A stream argument is a cudaStream_t (NULL = the legacy default stream).
 */
#ifndef FDMS_H
#define FDMS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fdms_cache fdms_cache;              /* opaque, owned by the library */

typedef enum {
  FDMS_OK = 0,
  FDMS_ERR_INVALID_ARG = 1,   /* bad argument, found on the host; nothing queued */
  FDMS_ERR_OUT_OF_BLOCKS = 2, /* the shared block pool ran out (device-latched) */
  FDMS_ERR_CUDA = 3,          /* a CUDA runtime call failed */
  FDMS_ERR_UNSUPPORTED = 4,   /* configuration the library has no kernel for */
  FDMS_ERR_DEVICE = 5,        /* other device-detected error (sequence longer than
                                 max_seq_len, a bounded wait that ran out) */
} fdms_status;

/* FDMS_KV_FP8_E4M3_BLOCK: E4M3 with one (K, V) scale pair per 64-slot store
 * block, from that block's own maxima (max(amax, 2^-126) / 448), fixed when the
 * block's 64th survivor arrives ("sealing"). Until then the store's partly
 * filled block stays bf16 in a per-head staging block, and the ring holds bf16
 * rows. Decode reads the sealed blocks as E4M3 with their own scales and the
 * staged block and the ring as bf16. Decode runs either mode (see
 * decode_ctas) with two running states per warp, one per tile kind. Per-head
 * clusters plan the sealed tiles the layer's previous decode saw before the
 * dependency wait (a sealed block never changes) and the staged and ring tiles
 * after it (the staged block changes in place); the global plan plans every
 * tile after the wait, with four warps per CTA. */
typedef enum { FDMS_KV_BF16 = 0, FDMS_KV_FP8_E4M3 = 1, FDMS_KV_FP8_E4M3_BLOCK = 2 } fdms_kv_dtype;

typedef struct {
  int num_layers;        /* L >= 1 */
  int max_batch;         /* sequence slots per layer, >= 1 */
  int num_q_heads;       /* Hq, a multiple of num_kv_heads */
  int num_kv_heads;      /* Hkv >= 1; G = Hq / Hkv in {1, 2, 4, 8} */
  int head_dim;          /* D in {64, 128} */
  int window;            /* W >= 0: always-visible recent tokens */
  int compact_period;    /* P >= 1: resolve out-of-window tokens P at a time */
  int max_seq_len;       /* tokens one (layer, seq) may hold, >= 1 */
  long long num_blocks;  /* 64-slot blocks in the shared pool; 0 = enough for
                            max_seq_len tokens in every (layer, seq, kv head) */
  fdms_kv_dtype kv_dtype;
  float softmax_scale;   /* 0 -> 1 / sqrt(head_dim) */
  int decode_ctas;       /* 0 -> automatic: a call whose (seq, kv head) pairs
                            can all hold a cluster of 8, 4 or 2 CTAs at once on
                            this device runs one cluster (of the largest such
                            size) per pair; other calls run
                            one plan over as many split CTAs as can be
                            resident on the device at once (two per SM for the
                            shapes here). > 0 -> always the plan, over this
                            many CTAs, at most that resident count */
} fdms_config;

typedef struct {
  long long tokens_appended;   /* sum over (layer, seq) of tokens appended */
  long long slots_store;       /* survivors in compact stores, all heads */
  long long slots_ring;        /* unresolved tokens in rings, all heads */
  long long blocks_used;       /* pool blocks handed out */
  long long blocks_free;       /* pool blocks left */
  long long bytes_compact;     /* (slots_store + slots_ring) * 2 * D * element bytes */
  long long bytes_dense_equiv; /* tokens_appended * num_kv_heads * 2 * D * element
                                  bytes: what a dense cache of the same dtype holds */
  long long bytes_reserved;    /* device bytes the cache allocated */
  long long fp8_saturations;   /* FP8: stored elements clipped to +-448 */
  long long slots_decoded;     /* cumulative slots (K row + V row each) read by
                                  decode calls: store slots plus ring slots */
  long long decode_calls;      /* decode calls so far */
  long long bytes_decoded;     /* cumulative K/V bytes of those slots (per-block FP8:
                                  sealed slots in E4M3, the others in bf16) */
  int error;                   /* sticky device error (an fdms_status), 0 if none */
} fdms_stats;

typedef struct {
  int num_tokens;  /* n: tokens appended to this (layer, seq, kv head) */
  int resolved;    /* r: positions resolved (store or dropped) */
  int store_len;   /* survivors in the compact store */
  int ring_len;    /* n - r: tokens in the ring */
} fdms_head_info;

/* Short English name of a status. Never NULL. */
const char* fdms_status_string(fdms_status s);

/* Create a cache on `device` and zero its state on `stream` (the call waits for
 * that work). *out receives the handle. Returns INVALID_ARG for a bad config,
 * UNSUPPORTED for a head_dim / group size without a kernel, CUDA when device
 * memory cannot be had (nothing is left allocated). */
fdms_status fdms_cache_create(const fdms_config* cfg, int device, void* stream,
                              fdms_cache** out);

/* Free everything the cache allocated. Synchronises the device first. NULL is OK. */
fdms_status fdms_cache_destroy(fdms_cache* cache);

/* Append tokens to sequences 0..batch-1 of `layer` and run eviction/compaction.
 *   n_new_dev     int32 [batch], device: tokens appended to each sequence,
 *                 0..max_new (values outside that range latch DEVICE).
 *   k_dev, v_dev  bf16 [batch][max_new][Hkv][D], device; row t of sequence b is
 *                 its position n_b + t.
 *   keep_dev      uint8 [batch][max_new][Hkv], device; nonzero = keep the slot
 *                 when it is resolved (the DMS decision).
 *   kv_scale_dev  FP8 only, optional: float [batch][Hkv][2] (K, V scales) used
 *                 for sequences that receive their first tokens in this call;
 *                 NULL = max(amax, 2^-126) / 448 of this call's values per head.
 *                 Must be NULL for a BF16 or per-block FP8 cache.
 * A sequence that would exceed max_seq_len is left unchanged and latches DEVICE.
 * A head whose survivors do not fit in the pool is left unchanged and latches
 * OUT_OF_BLOCKS. */
fdms_status fdms_append_evict(fdms_cache* cache, int layer, int batch,
                              const int32_t* n_new_dev, int max_new,
                              const void* k_dev, const void* v_dev,
                              const uint8_t* keep_dev, const float* kv_scale_dev,
                              void* stream);

/* Decode attention of sequences 0..batch-1 of `layer`:
 *   q_dev    bf16 [batch][Hq][D], device.
 *   out_dev  bf16 [batch][Hq][D], device: softmax(scale * q K_S^T) V_S over the
 *            visible set S of the query head's kv head, rounded to nearest even.
 *            A head with no visible token gets zeros.
 * The split partials live in the cache's workspace, so two decode calls on one
 * cache must not overlap (queue them on one stream). */
fdms_status fdms_decode_attn(fdms_cache* cache, int layer, int batch,
                             const void* q_dev, void* out_dev, void* stream);

/* fdms_decode_attn with fp32 output and, if lse_dev is not NULL, the natural
 * log of the softmax denominator per query head (float [batch][Hq], -inf for an
 * empty head): log sum_{j in S} exp(scale * q.k_j). */
fdms_status fdms_decode_attn_f32(fdms_cache* cache, int layer, int batch,
                                 const void* q_dev, float* out_dev, float* lse_dev,
                                 void* stream);

/* Bytes of the library's fixed decode scratch array (one per device). */
#define FDMS_STATIC_SCRATCH_BYTES (4u << 20)

/* fdms_decode_attn for callers that cannot allocate device memory. The pages
 * describe nothing like it: it exists for code that must not call cudaMalloc
 * (or anything that allocates, torch's allocator included) on its decode path,
 * for example a runtime whose device memory is all handed out up front by
 * another owner, or a loop that may not allocate once it is running.
 * Same arguments, layouts and result as fdms_decode_attn. The split partials,
 * which fdms_decode_attn keeps in workspace the cache allocated, go instead
 * into one static array of FDMS_STATIC_SCRATCH_BYTES compiled into the library;
 * every device that loads the library holds that array until the process exits.
 *   - Needs (split warps + batch x Hkv) x G x (4 D + 8) bytes plus
 *     4 x batch x Hkv bytes of merge counters, each part rounded up to 256
 *     (at most one partial per split warp and head it shares with another
 *     warp; 4 to 6 split warps per decode CTA), or none for a call that runs in
 *     per-head clusters (see decode_ctas); a call that needs more than the
 *     array returns FDMS_ERR_INVALID_ARG and queues nothing. The call clears
 *     the counters on its stream before its kernel; every other value it reads
 *     from the array it first writes itself.
 *   - The first call on a device looks up the array's device address (a
 *     runtime query, no allocation); make that first call before any stream
 *     capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind: calls whose work overlaps on the GPU (different streams, or
 *     different caches at once) race. Queue them on one stream.
 * Allocates nothing and calls no allocating routine. */
fdms_status fdms_decode_attn_noalloc(fdms_cache* cache, int layer, int batch,
                                     const void* q_dev, void* out_dev, void* stream);

/* How a decode call of `batch` sequences would run on this cache (no device
 * work): *cluster_ctas_out receives the CTAs of the thread-block cluster per
 * (seq, kv head) (2, 4 or 8), or 0 when the call runs the global plan, whose
 * split grid (CTAs) goes to *split_ctas_out. Either pointer may be NULL.
 * INVALID_ARG for a NULL cache or batch outside 1..max_batch. */
fdms_status fdms_decode_layout(fdms_cache* cache, int batch, int* cluster_ctas_out,
                               int* split_ctas_out);

/* Gather the counters on `stream` and wait for them. */
fdms_status fdms_cache_stats(fdms_cache* cache, fdms_stats* host_out, void* stream);

/* Copy one head's contents to host memory, in position order: entries
 * [0, store_len) are the compact store, [store_len, store_len + ring_len) the
 * ring. Waits for `stream` first.
 *   capacity     entries the host buffers hold (INVALID_ARG if too few).
 *   pos_host     int32 [capacity]: token positions.
 *   keep_host    uint8 [capacity]: keep bits (1 for store entries).
 *   k_host/v_host  [capacity][D * element bytes]: stored payload (bf16 or E4M3).
 *                FDMS_KV_FP8_E4M3_BLOCK: [capacity][2 D] bytes; a sealed entry
 *                holds its D E4M3 codes in the first D bytes (the rest zero), a
 *                staged or ring entry its D bf16 values.
 *   scale_host   float [capacity][2]: (K, V) scale applied to each entry
 *                (1.0 for BF16; 0 for the bf16 entries of FDMS_KV_FP8_E4M3_BLOCK).
 *   info_host    counts, always filled.
 * Any pointer but info_host may be NULL to skip it. */
fdms_status fdms_cache_read_head(fdms_cache* cache, int layer, int seq, int kv_head,
                                 int capacity, int32_t* pos_host, uint8_t* keep_host,
                                 void* k_host, void* v_host, float* scale_host,
                                 fdms_head_info* info_host, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FDMS_H */

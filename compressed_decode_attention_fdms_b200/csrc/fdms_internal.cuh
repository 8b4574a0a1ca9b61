// Internal layout of the compact KV cache and device helpers shared by the
// kernels. Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fdms.h"

namespace fdms {

constexpr int kBlockSlots = 64;        // slots per pool block (= FP8 scale granularity)
constexpr int kMaxGroup = 8;

// Device-side counters and the sticky error word.
struct DevCounters {
  unsigned long long blocks_next;      // bump allocator over the pool
  unsigned long long saturations;      // FP8 elements clipped on write
  int error;                           // first error code latched (fdms_status)
  int pad;
  unsigned long long slots_decoded;    // cumulative units scanned by decode calls
  unsigned long long decode_calls;
  unsigned long long bytes_decoded;    // cumulative K/V bytes those units hold
  // stats scratch (filled by the stats kernel)
  unsigned long long tokens, slots_store, slots_ring, slots_sealed;
};

// Everything a kernel needs to find a head's data. Passed by value.
//
// Head index hi = (layer * Bmax + seq) * Hkv + kv_head.
//   block_table[hi * max_blocks + j]   physical block of the head's j-th store block
//   bt_scale[(hi * max_blocks + j) * 2 + {0,1}]  K / V scale of that block
//   store_len[hi], tok_n[hi], tok_r[hi]
//   ring:      hi * 2 * R * RB bytes; K rows [R][RB] then V rows [R][RB]
//              (position p lives in slot p % R; R is a multiple of 64)
//   ring_keep: hi * Rpad bytes
//   head_scale[hi * 2 + {0,1}]         FP8 scale of K / V
//   per-block FP8 (blk): stage: hi * 2 * 64 * 2D bytes, bf16 K rows [64][2D]
//              then V rows, the store's partly filled block; stage_pos[hi * 64
//              + row] their positions; ring rows are bf16 too (RBR = 2D)
// Pool block b: K rows [64][RB] at pool + b * 2 * 64 * RB, V rows right after;
//   blk_pos[b * 64 + row] is the token position of each slot.
struct CacheView {
  uint8_t* pool;
  int32_t* blk_pos;
  float* bt_scale;
  int32_t* block_table;
  int32_t* store_len;
  int32_t* tok_n;
  int32_t* tok_r;
  uint8_t* ring;
  uint8_t* ring_keep;
  float* head_scale;
  DevCounters* ctr;
  uint8_t* stage;         // per-block FP8 only
  int32_t* stage_pos;     // per-block FP8 only
  long long num_blocks;
  int L, Bmax, Hq, Hkv, G, D, RB, W, P, R, Rpad, max_blocks, max_seq_len;
  int RBR;                // bytes of a ring row (RB, or 2 D for per-block FP8)
  int fp8;
  int blk;                // per-block FP8 scales (FDMS_KV_FP8_E4M3_BLOCK)
  float softmax_scale;
  // bytes every decode tile stage expects beyond its copies: 0, or 16 when
  // FDMS_TEST_STALL_COPIES is set at cache creation (failure-detection tests:
  // the copies land but no stage completes, so every stage wait runs out)
  uint32_t stall_tx;
};

// Row layout inside a 64-row page (a store block, or 64 ring slots): the 16-byte
// chunks of row r are stored XOR-permuted by r, so that the decode kernel's
// matrix loads from shared memory (ldmatrix: eight consecutive rows, one
// 16-byte chunk each) touch every bank once. Rows keep their page-row index r
// in shared memory, so the permutation survives a straight bulk copy. The
// permutation depends on r mod 8 only: 128- and 256-byte rows XOR the chunk
// index with r mod 8 (eight rows, eight distinct 16-byte bank groups); 64-byte
// rows, two to a 128-byte line, XOR it with (r / 2) mod 4. K and V rows use
// the same permutation.
__host__ __device__ inline int swz_chunk(int RB, bool is_v, int row, int chunk) {
  (void)is_v;
  if (RB == 64) return chunk ^ ((row >> 1) & 3);
  return chunk ^ (row & 7);
}
// Byte offset inside a row of the logical byte b (the chunk permutation keeps
// the byte's place inside its chunk).
__host__ __device__ inline int swz_byte(int RB, bool is_v, int row, int b) {
  return swz_chunk(RB, is_v, row, b >> 4) * 16 + (b & 15);
}

__host__ __device__ inline long long head_index(const CacheView& c, int layer, int seq, int h) {
  return ((long long)layer * c.Bmax + seq) * c.Hkv + h;
}
__host__ __device__ inline uint8_t* block_k(const CacheView& c, long long blk) {
  return c.pool + blk * 2LL * kBlockSlots * c.RB;
}
__host__ __device__ inline uint8_t* block_v(const CacheView& c, long long blk) {
  return block_k(c, blk) + (long long)kBlockSlots * c.RB;
}
__host__ __device__ inline uint8_t* ring_k(const CacheView& c, long long hi) {
  return c.ring + hi * 2LL * c.R * c.RBR;
}
__host__ __device__ inline uint8_t* ring_v(const CacheView& c, long long hi) {
  return ring_k(c, hi) + (long long)c.R * c.RBR;
}
__host__ __device__ inline uint8_t* stage_k(const CacheView& c, long long hi) {
  return c.stage + hi * 2LL * kBlockSlots * (2 * c.D);
}
__host__ __device__ inline uint8_t* stage_v(const CacheView& c, long long hi) {
  return stage_k(c, hi) + (long long)kBlockSlots * (2 * c.D);
}

// Decode workspace: the split partials (warp v's partial of head h at v + h).
struct DecodeWork {
  float* part_o;          // [max_parts][G][D], unnormalised sum of p * v
  float* part_ml;         // [max_parts][G][2]: running max (log2 domain) and sum
  int max_parts;
  int max_ctas;
  int4* snap;             // [2][L * Bmax * Hkv]: per head, (store_len, n, r, 0) as a
                          // decode of it saw them; two copies, so that the kernel
                          // that writes one never races its own reads of the other
  int4* snap_rd;          // this call's copies (set per call): the one it reads
  int4* snap_wr;          // and the one it writes for the next decode of the layer
  int* head_cnt;          // [Bmax * Hkv]: partials of a head merged so far (global
                          // plan); back to 0 once merged
};

// Workspace of the bulk (prefill) append, per (seq, kv head) of the call.
constexpr int kChunkPositions = 1024;  // positions per chunk of the bulk append
constexpr int kHdrInts = 16;
struct AppendWork {
  int* counts;            // [heads][max_chunks]: survivors per chunk, then their prefix
  int* hdr;               // [heads][kHdrInts]: state before the call, allocation, scales
  unsigned* amax;         // [heads][2]: bits of max |x| over the call's K / V (FP8)
  int max_chunks;
};

// K/V bytes a decode call reads for a head of store length len and ring
// positions [r, n): one K row and one V row per slot, of D elements (per-block
// FP8: the sealed blocks' rows in E4M3, the staged block's and the ring's in bf16)
__device__ inline unsigned long long head_kv_bytes(const CacheView& c, int len, int n, int r) {
  const unsigned long long row = 2ull * c.RB;
  if (!c.blk) return (unsigned long long)(len + (n - r)) * row;
  const int sealed = len / kBlockSlots * kBlockSlots;
  return (unsigned long long)sealed * row + (unsigned long long)(len - sealed + (n - r)) * 2 * row;
}

__device__ inline void latch_error(DevCounters* ctr, int code) {
  atomicCAS(&ctr->error, 0, code);
}

// ---------------------------------------------------------------- numerics
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// f32 -> bf16 bits, round to nearest even
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
  return r;
}

// two E4M3 codes (low byte first) -> two f32, exact (via f16x2)
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t two) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(two));
  float lo, hi;
  asm("{.reg .f16 a, b;\n mov.b32 {a, b}, %2;\n cvt.f32.f16 %0, a;\n cvt.f32.f16 %1, b;}"
      : "=f"(lo), "=f"(hi) : "r"(h));
  return make_float2(lo, hi);
}

// two f32 -> two E4M3 codes (x0 in the low byte), round to nearest even, satfinite
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float x0, float x1) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
  return r;
}

// packed fp32 fused multiply-add (sm_100): d = a * b + c on both lanes
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n"
      " mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rc, {%6, %7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------- bulk copy + mbarrier (PTX)
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
// raise the transaction count of the current phase without arriving (the
// arrival comes later)
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;"
               ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
// returns true once the phase with the given parity has completed
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p;\n"
      "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p; }"
      : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// global -> shared bulk copy into this CTA's own shared memory, completion counted on `bar`
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst_smem)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

// 4-byte global -> shared copy in the background (LDGSTS), and an arrival on
// `bar` once every such copy this thread issued has landed (the barrier counts
// one arrival per thread that calls it)
__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst_smem)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}
// atomic add with release and acquire semantics at GPU scope: writes this
// thread made (or saw, e.g. through a warp barrier) before it are visible to
// a thread that reads its result, and that thread sees them after it
__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

// add without a result, with release semantics at GPU scope (the writes this
// thread made or saw before it are visible to whoever acquires the sum)
__device__ __forceinline__ void red_add_release(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Programmatic dependent launch: wait for the preceding grid's memory, and let
// the next grid start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;");
}

}  // namespace fdms

// Host-side cache object.
struct fdms_cache {
  fdms_config cfg;
  int device;
  int num_sms;
  fdms::CacheView view;
  fdms::DecodeWork work;
  fdms::AppendWork awork;
  size_t bytes_reserved;
  // allocations (freed at destroy)
  void* allocs[32];
  int nallocs;
  int decode_ctas;        // split grid used
  int ctas_per_sm;
  int ranges_per_cta;     // warps per split CTA (one unit range each)
  int cluster_ok;         // the per-head cluster decode mode can be launched
  int max_clusters[4];    // clusters of 2, 4, 8 CTAs (index 1..3) resident at once
  int plan_ctas_per_sm;   // global-plan split CTAs that fit on one SM
  // Kernels queued on the cache, numbered from 1 in launch order. A kernel
  // that lets its successor start only after its own dependency wait ("waits
  // first": every decode kernel, the bulk and small appends) has seen every
  // kernel before it finish when it passes that wait; the decode-step append
  // lets its successor start at once. So when a new kernel starts, every
  // kernel queued before the latest "waits first" one has finished: a head's
  // state may be read before the dependency wait only if its last writer is
  // one of those.
  long long launches;         // kernels queued so far
  long long last_wait_first;  // number of the latest "waits first" kernel, 0: none
  long long* append_at;       // [L]: number of the last append kernel to the layer
  long long* decode_at;       // [L]: number of the last decode kernel of the layer
  long long* tokens_since;    // [L]: tokens per sequence appended since that decode
  int* decode_batch;          // [L]: batch of that decode
  long long* decode_count;    // [L]: decode calls of the layer so far (snapshot copy)
};

// Number a kernel just queued; `waits_first`: it lets its successor start only
// after its own dependency wait.
inline long long fdms_log_launch(fdms_cache* c, bool waits_first) {
  const long long n = ++c->launches;
  if (waits_first) c->last_wait_first = n;
  return n;
}
// Kernel number n (0: none) has certainly finished when the next kernel starts.
inline bool fdms_log_finished(const fdms_cache* c, long long n) {
  return n < c->last_wait_first;
}

// Record a device allocation of the cache (freed at destroy). Frees `p` and
// returns false when the table is full.
inline bool fdms_track(fdms_cache* c, void* p, size_t bytes) {
  if (c->nallocs >= (int)(sizeof(c->allocs) / sizeof(c->allocs[0]))) {
    cudaFree(p);
    return false;
  }
  c->allocs[c->nallocs++] = p;
  c->bytes_reserved += bytes;
  return true;
}

// launchers (defined in their .cu files)
fdms_status fdms_launch_append(fdms_cache* c, int layer, int batch, const int32_t* n_new,
                               int max_new, const void* k, const void* v, const uint8_t* keep,
                               const float* kv_scale, cudaStream_t s);
fdms_status fdms_launch_decode(fdms_cache* c, int layer, int batch, const void* q, void* out,
                               int out_f32, float* lse, cudaStream_t s);
fdms_status fdms_decode_setup(fdms_cache* c);
fdms_status fdms_append_setup(fdms_cache* c);

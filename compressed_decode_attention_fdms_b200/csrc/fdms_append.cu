// Append + evict + compact.
//
// What it applies (FastDMS announcement, aiwitness.kr/community/1t3vlrx, the
// paragraphs on DMS per-head token eviction and on the compact store that
// physically reclaims evicted slots, with its staging area):
//   1. new tokens of the call take positions n0 .. n1-1;
//   2. if at least P out-of-window tokens are unresolved, all positions
//      r0 .. n1-W-1 are resolved now: in position order, those with keep = 1
//      are appended to the head's compact store, the rest are dropped;
//   3. the still-unresolved new tokens are written to the ring (staging).
// Resolution is a stable stream compaction (warp ballot of the keep bits, a
// popcount prefix inside each warp, a scan of warp totals), so survivors keep
// their order. Store blocks for all survivors of a head are reserved in one
// step before any row is written; if the pool cannot cover them the head is
// left unchanged, the pool counter does not move, and FDMS_ERR_OUT_OF_BLOCKS is
// latched.
//
// Three paths, one result: decode steps (k_append_step: a warp per head, the
// loads ordered for latency), calls of up to 16 tokens per sequence
// (k_append_small: a warp per head) and bulk calls such as prefill (four
// launches spread over many CTAs per head, below). A per-block FP8 cache has
// its own two (k_append_block, a warp per head; k_append_block_cta, a CTA per
// head for calls of 64 tokens or more), at the end of this file.
//
// FP8 cache: a sequence's first append fixes each head's K and V scales
// (max(amax, 2^-126) / 448 of the call's values, or the caller's); every new
// row is stored as e4m3_rne_satfinite(fp32(x) / scale) with the quotient
// correctly rounded in IEEE fp32 and the rounding to E4M3 by the hardware
// conversion.
#include <algorithm>

#include "fdms_internal.cuh"

namespace fdms {
namespace {

constexpr int kAppendThreads = 256;
constexpr int kWarps = kAppendThreads / 32;

__device__ __forceinline__ float block_max(float x, float* red) {
  for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = x;
  __syncthreads();
  float m = red[0];
  for (int i = 1; i < kWarps; ++i) m = fmaxf(m, red[i]);
  return m;
}

// Blocks [base, base + need) of the pool for one head, or -1 when the pool
// cannot cover them. The counter never moves past num_blocks: a request that
// does not fit leaves it as it was, so a later, smaller request can still be
// served and the count of blocks handed out stays exact. A compare-and-swap
// loop: warps of one kernel rarely contend (a decode step takes a new block
// about once per 64 kept tokens of a head). Gives up (-1) after a bounded
// number of lost races.
__device__ long long take_blocks(DevCounters* ctr, unsigned long long need, long long num_blocks) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(&ctr->blocks_next);
  for (int it = 0; it < (1 << 16); ++it) {
    if (cur + need > (unsigned long long)num_blocks) return -1;
    const unsigned long long prev = atomicCAS(&ctr->blocks_next, cur, cur + need);
    if (prev == cur) return (long long)cur;
    cur = prev;
  }
  return -1;
}

// x / s in IEEE binary32, rounded to nearest even, for finite x and a normal
// s > 0, given r = RN(1/s): q = RN(x r), then one correction with the exact
// residual x - q s (one FMA). This is Markstein's division (IBM J. Res. Dev.
// 34(1), 1990): with r correctly rounded and q within an ulp of x / s, the
// corrected quotient is the correctly rounded one. Where the quotient
// overflows, q itself is returned (both saturate when converted); quotients
// below the normal range convert to an E4M3 zero whatever their rounding.
__device__ __forceinline__ float div_rn(float x, float s, float r) {
  const float q = x * r;
  const float q1 = fmaf(fmaf(-q, s, x), r, q);
  return isfinite(q1) ? q1 : q;
}

// The reciprocal div_rn takes: RN(1 / scale), or 0 where 1 / scale might
// overflow (scale < 1e-30), which sends quantise8 to plain division. Computed
// once per scale, not per vector.
__device__ __forceinline__ float quant_recip(float scale) {
  return scale < 1.0e-30f ? 0.f : __frcp_rn(scale);
}

// 8 bf16 (one 16-byte vector) / scale -> 8 E4M3 codes; counts clipped values.
// r = quant_recip(scale).
__device__ __forceinline__ uint2 quantise8(uint4 x, float scale, float r, unsigned& sat) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  float f[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = bf16lo_to_f32(w[j]);
    f[2 * j + 1] = bf16hi_to_f32(w[j]);
  }
  if (r != 0.f) {   // one branch for the vector: the common path has no division
#pragma unroll
    for (int t = 0; t < 8; ++t) f[t] = div_rn(f[t], scale, r);
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) f[t] = __fdiv_rn(f[t], scale);
  }
#pragma unroll
  for (int t = 0; t < 8; ++t) sat += fabsf(f[t]) > 448.0f ? 1u : 0u;
  const uint32_t lo = (uint32_t)f32x2_to_e4m3x2(f[0], f[1]) |
                      ((uint32_t)f32x2_to_e4m3x2(f[2], f[3]) << 16);
  const uint32_t hi = (uint32_t)f32x2_to_e4m3x2(f[4], f[5]) |
                      ((uint32_t)f32x2_to_e4m3x2(f[6], f[7]) << 16);
  return make_uint2(lo, hi);
}

// Copy one 16-byte vector `vec` (8 bf16 values) of an input row into row `row`
// of a cache page (quantising in FP8 mode, where it becomes 8 bytes), at its
// place in the page's chunk permutation.
template <bool FP8>
__device__ __forceinline__ void put_input_vec(uint8_t* dst_row, const uint16_t* src_row, int vec,
                                              float scale, float r, unsigned& sat, int RB,
                                              bool is_v, int row) {
  const uint4 x = *reinterpret_cast<const uint4*>(src_row + vec * 8);
  if constexpr (FP8) {
    *reinterpret_cast<uint2*>(dst_row + swz_byte(RB, is_v, row, vec * 8)) =
        quantise8(x, scale, r, sat);
  } else {
    *reinterpret_cast<uint4*>(dst_row + swz_byte(RB, is_v, row, vec * 16)) = x;
  }
}

// Move one vector of a cached row between pages (ring slot -> store row).
template <bool FP8>
__device__ __forceinline__ void move_vec(uint8_t* dst_row, int dst_r, const uint8_t* src_row,
                                         int src_r, int vec, int RB, bool is_v) {
  if constexpr (FP8) {
    *reinterpret_cast<uint2*>(dst_row + swz_byte(RB, is_v, dst_r, vec * 8)) =
        *reinterpret_cast<const uint2*>(src_row + swz_byte(RB, is_v, src_r, vec * 8));
  } else {
    *reinterpret_cast<uint4*>(dst_row + swz_byte(RB, is_v, dst_r, vec * 16)) =
        *reinterpret_cast<const uint4*>(src_row + swz_byte(RB, is_v, src_r, vec * 16));
  }
}

// ================================================================ bulk append
// Calls with more than kSmallMax new tokens per sequence (prefill): four
// launches, the data-moving ones spread over many CTAs per (seq, kv head),
// with the same result as the warp paths.
//   1. k_bulk_count (head x chunk): survivors of each chunk of kChunkPositions
//      of the positions resolved now; on a sequence's first FP8 append, the
//      call's max |K| and |V| (atomicMax on the bits of non-negative floats).
//   2. k_bulk_alloc (one CTA for the call): exclusive prefix of the chunk
//      counts per head, the FP8 scales, the store blocks of all heads reserved
//      in head order, and the heads' new lengths; the state before the call
//      goes to the workspace header, which the next two kernels read instead.
//   3. k_bulk_write (head x chunk): the chunk's survivors to the store, in
//      order, at len0 + prefix + rank (warp ballot/popc, scan of warp totals).
//   4. k_bulk_ring (head): the still-unresolved new tokens to the ring, once
//      every ring row that (3) resolves has been read.
enum : int { kHdrM, kHdrN0, kHdrR0, kHdrLen0, kHdrN1, kHdrR1, kHdrNb0, kHdrStatus, kHdrLen1,
             kHdrSk, kHdrSv };
enum : int { kBulkGo = 0, kBulkSkip = 1 };

struct BulkIn {
  const int32_t* n_new;
  const uint16_t* k_in;
  const uint16_t* v_in;
  const uint8_t* keep_in;
  const float* kv_scale;
  int batch, max_new, layer;
};

// max |x| over rows [r_lo, r_hi) of D bf16 values (row stride `stride`),
// CTA-wide; eight 16-byte loads in flight per thread
__device__ float rows_amax_range(const uint16_t* base, int r_lo, int r_hi, int D, long long stride,
                                 float* red) {
  float a = 0.0f;
  const int vpr = D / 8;
  const long long nv = (long long)(r_hi - r_lo) * vpr;
  for (long long i0 = threadIdx.x; i0 < nv; i0 += 8LL * kAppendThreads) {
    uint4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const long long i = i0 + (long long)u * kAppendThreads;
      x[u] = i < nv ? *reinterpret_cast<const uint4*>(base + (r_lo + i / vpr) * stride +
                                                       (i % vpr) * 8)
                    : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a = fmaxf(a, fabsf(bf16lo_to_f32(w[j])));
        a = fmaxf(a, fabsf(bf16hi_to_f32(w[j])));
      }
    }
  }
  return block_max(a, red);
}

template <bool FP8>
__global__ void __launch_bounds__(kAppendThreads)
k_bulk_count(CacheView c, AppendWork aw, BulkIn in) {
  __shared__ float s_red[kWarps];
  pdl_wait();                 // the previous kernel's writes are visible from here on
  pdl_launch_dependents();
  const int hid = blockIdx.x, ch = blockIdx.y, nch = gridDim.y, tid = threadIdx.x;
  const int b = hid / c.Hkv, h = hid % c.Hkv;
  const long long hi = head_index(c, in.layer, b, h);
  const int m = in.n_new[b];
  const int n0 = c.tok_n[hi], r0 = c.tok_r[hi];
  int cnt = 0;
  if (m > 0 && m <= in.max_new && (long long)n0 + m <= c.max_seq_len) {
    const int n1 = n0 + m;
    const int r1 = (n1 - c.W - r0 >= c.P) ? n1 - c.W : r0;
    const uint8_t* rkeep = c.ring_keep + hi * c.Rpad;
    const uint8_t* keep_rows = in.keep_in + (long long)b * in.max_new * c.Hkv + h;
    const int p_lo = r0 + ch * kChunkPositions, p_hi = min(r1, p_lo + kChunkPositions);
    for (int base = p_lo; base < p_hi; base += kAppendThreads) {
      const int p = base + tid;
      int keep = 0;
      if (p < p_hi)
        keep = p < n0 ? (rkeep[p % c.R] != 0) : (keep_rows[(long long)(p - n0) * c.Hkv] != 0);
      cnt += __syncthreads_count(keep);
    }
    if constexpr (FP8) {
      if (n0 == 0 && !in.kv_scale) {   // rows [ch rpc, (ch + 1) rpc) of the call
        const long long in_stride = (long long)c.Hkv * c.D;
        const long long off = ((long long)b * in.max_new * c.Hkv + h) * c.D;
        const int rpc = (m + nch - 1) / nch;
        const int lo = min(m, ch * rpc), hi_r = min(m, lo + rpc);
        const float ak = rows_amax_range(in.k_in + off, lo, hi_r, c.D, in_stride, s_red);
        const float av = rows_amax_range(in.v_in + off, lo, hi_r, c.D, in_stride, s_red);
        if (tid == 0) {
          atomicMax(&aw.amax[hid * 2], __float_as_uint(ak));
          atomicMax(&aw.amax[hid * 2 + 1], __float_as_uint(av));
        }
      }
    }
  }
  if (tid == 0) aw.counts[(long long)hid * aw.max_chunks + ch] = cnt;
}

constexpr int kAllocThreads = 1024;
constexpr int kAllocWarps = kAllocThreads / 32;
constexpr int kMaxCallHeads = 4096;   // max_batch x num_kv_heads of a supported cache
constexpr int kAllocPer = kMaxCallHeads / kAllocThreads;

// Dynamic shared memory of k_bulk_alloc for a call of `heads` heads: blocks
// needed, first block, first new block-table entry, FP8 scales (K, V).
inline size_t bulk_alloc_smem(int heads) { return (size_t)heads * 5 * sizeof(int); }

// One CTA for every head of the call, in three phases:
//   1. a thread per head (heads tid, tid + 1024, ...): exclusive prefix of the
//      chunk counts, FP8 scales, the state before the call and after it (into
//      the head's header, for the kernels after this one; the thread keeps it
//      in registers), and the pool blocks the head needs;
//   2. the blocks of all heads reserved at once, in head order; when the pool
//      cannot cover them all, heads are served first-fit in head order, so a
//      head that does not fit leaves the pool to the heads after it;
//   3. the owning thread writes the head's new lengths, or the error for a
//      head that got no blocks (left unchanged); then a warp per head writes
//      the block-table entries and their scales.
// Allocations of different kernels never overlap (each runs after its
// dependency wait), so inside this kernel the pool counter has one writer.
template <bool FP8>
__global__ void __launch_bounds__(kAllocThreads)
k_bulk_alloc(CacheView c, AppendWork aw, BulkIn in, int nch, int heads) {
  extern __shared__ int s_alloc[];
  int* s_need = s_alloc;               // blocks a head needs; -1: nothing to do
  int* s_blk = s_need + heads;         // first block handed out; -1: none
  int* s_nb0 = s_blk + heads;          // first new block-table entry
  float* s_sk = reinterpret_cast<float*>(s_nb0 + heads);
  float* s_sv = s_sk + heads;
  __shared__ int s_wsum[kAllocWarps];
  __shared__ long long s_base;
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  // ---- phase 1
  int st_len1[kAllocPer], st_n1[kAllocPer], st_r1[kAllocPer];
#pragma unroll
  for (int i = 0; i < kAllocPer; ++i) {
    const int hid = tid + i * kAllocThreads;
    st_len1[i] = st_n1[i] = st_r1[i] = 0;
    if (hid >= heads) continue;
    const int b = hid / c.Hkv, h = hid % c.Hkv;
    const long long hi = head_index(c, in.layer, b, h);
    int* hd = aw.hdr + (long long)hid * kHdrInts;
    const int m = in.n_new[b];
    const int n0 = c.tok_n[hi], r0 = c.tok_r[hi], len0 = c.store_len[hi];
    unsigned ak_bits = 0, av_bits = 0;
    if constexpr (FP8) {
      ak_bits = aw.amax[hid * 2];
      av_bits = aw.amax[hid * 2 + 1];
      aw.amax[hid * 2] = 0u;   // ready for the next call
      aw.amax[hid * 2 + 1] = 0u;
    }
    if (m < 0 || m > in.max_new || (long long)n0 + m > c.max_seq_len || m == 0) {
      if (m != 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
      hd[kHdrStatus] = kBulkSkip;
      s_need[hid] = -1;
      continue;
    }
    const int n1 = n0 + m;
    const int r1 = (n1 - c.W - r0 >= c.P) ? n1 - c.W : r0;
    // exclusive prefix of the chunk counts, eight loads in flight
    int* cnt = aw.counts + (long long)hid * aw.max_chunks;
    int running = 0;
    for (int base = 0; base < nch; base += 8) {
      int x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = base + u < nch ? cnt[base + u] : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (base + u < nch) cnt[base + u] = running;
        running += x[u];
      }
    }
    const int len1 = len0 + running;
    // FP8 scales: a sequence's first append fixes them
    float sk = 1.0f, sv = 1.0f;
    if constexpr (FP8) {
      if (n0 == 0) {
        if (in.kv_scale) {
          sk = in.kv_scale[((long long)b * c.Hkv + h) * 2];
          sv = in.kv_scale[((long long)b * c.Hkv + h) * 2 + 1];
        } else {
          sk = __fdiv_rn(fmaxf(__uint_as_float(ak_bits), 1.17549435e-38f), 448.0f);
          sv = __fdiv_rn(fmaxf(__uint_as_float(av_bits), 1.17549435e-38f), 448.0f);
        }
        c.head_scale[hi * 2] = sk;
        c.head_scale[hi * 2 + 1] = sv;
      } else {
        sk = c.head_scale[hi * 2];
        sv = c.head_scale[hi * 2 + 1];
      }
    }
    const int nb0 = (len0 + kBlockSlots - 1) / kBlockSlots;
    const int nb1 = (len1 + kBlockSlots - 1) / kBlockSlots;
    hd[kHdrM] = m;
    hd[kHdrN0] = n0;
    hd[kHdrR0] = r0;
    hd[kHdrLen0] = len0;
    hd[kHdrN1] = n1;
    hd[kHdrR1] = r1;
    hd[kHdrNb0] = nb0;
    hd[kHdrLen1] = len1;
    hd[kHdrStatus] = kBulkGo;
    hd[kHdrSk] = __float_as_int(sk);
    hd[kHdrSv] = __float_as_int(sv);
    s_need[hid] = nb1 - nb0;
    s_nb0[hid] = nb0;
    s_sk[hid] = sk;
    s_sv[hid] = sv;
    st_len1[i] = len1;
    st_n1[i] = n1;
    st_r1[i] = r1;
  }
  __syncthreads();

  // ---- phase 2: exclusive prefix of the needs in head order (thread tid
  // holds heads tid * kAllocPer .. tid * kAllocPer + kAllocPer - 1)
  int mine[kAllocPer], sum = 0;
#pragma unroll
  for (int i = 0; i < kAllocPer; ++i) {
    const int hid = tid * kAllocPer + i;
    mine[i] = hid < heads ? max(s_need[hid], 0) : 0;
    sum += mine[i];
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  int excl = incl - sum, total = 0;
  for (int i = 0; i < kAllocWarps; ++i) {
    if (i < warp) excl += s_wsum[i];
    total += s_wsum[i];
  }
  if (tid == 0) {
    const long long cur = (long long)c.ctr->blocks_next;
    if (cur + total <= c.num_blocks) {
      s_base = cur;
      c.ctr->blocks_next = (unsigned long long)(cur + total);
    } else {
      s_base = -1;
    }
  }
  __syncthreads();
  if (s_base >= 0) {
#pragma unroll
    for (int i = 0; i < kAllocPer; ++i) {
      const int hid = tid * kAllocPer + i;
      if (hid < heads) s_blk[hid] = (int)(s_base + excl);
      excl += mine[i];
    }
  } else if (tid == 0) {   // the pool falls short: first fit in head order
    long long cur = (long long)c.ctr->blocks_next;
    for (int hid = 0; hid < heads; ++hid) {
      const int need = s_need[hid];
      if (need <= 0) {
        s_blk[hid] = (int)cur;
      } else if (cur + need <= c.num_blocks) {
        s_blk[hid] = (int)cur;
        cur += need;
      } else {
        s_blk[hid] = -1;
      }
    }
    c.ctr->blocks_next = (unsigned long long)cur;
  }
  __syncthreads();

  // ---- phase 3: lengths (owning thread), then block tables (warp per head)
#pragma unroll
  for (int i = 0; i < kAllocPer; ++i) {
    const int hid = tid + i * kAllocThreads;
    if (hid >= heads || s_need[hid] < 0) continue;
    const long long hi = head_index(c, in.layer, hid / c.Hkv, hid % c.Hkv);
    if (s_blk[hid] < 0) {
      latch_error(c.ctr, FDMS_ERR_OUT_OF_BLOCKS);
      aw.hdr[(long long)hid * kHdrInts + kHdrStatus] = kBulkSkip;
      continue;
    }
    c.store_len[hi] = st_len1[i];
    c.tok_n[hi] = st_n1[i];
    c.tok_r[hi] = st_r1[i];
  }
  for (int hid = warp; hid < heads; hid += kAllocWarps) {
    const int need = s_need[hid];
    const long long base_blk = s_blk[hid];
    if (need <= 0 || base_blk < 0) continue;
    const long long hi = head_index(c, in.layer, hid / c.Hkv, hid % c.Hkv);
    const int nb0 = s_nb0[hid];
    const float sk = s_sk[hid], sv = s_sv[hid];
    int32_t* bt = c.block_table + hi * c.max_blocks;
    float* bts = c.bt_scale + hi * c.max_blocks * 2;
    for (int j = lane; j < need; j += 32) {
      bt[nb0 + j] = (int32_t)(base_blk + j);
      bts[2 * (nb0 + j)] = sk;
      bts[2 * (nb0 + j) + 1] = sv;
    }
  }
}

template <bool FP8>
__global__ void __launch_bounds__(kAppendThreads)
k_bulk_write(CacheView c, AppendWork aw, BulkIn in) {
  __shared__ int s_warp[kWarps];
  __shared__ int s_src[kChunkPositions];   // survivors of the chunk, in order
  __shared__ int s_total;
  pdl_wait();
  pdl_launch_dependents();
  const int hid = blockIdx.x, ch = blockIdx.y, tid = threadIdx.x, warp = tid / 32,
            lane = tid % 32;
  const int* hd = aw.hdr + (long long)hid * kHdrInts;
  if (hd[kHdrStatus] != kBulkGo) return;
  const int n0 = hd[kHdrN0], r0 = hd[kHdrR0], len0 = hd[kHdrLen0], r1 = hd[kHdrR1];
  const float sk = __int_as_float(hd[kHdrSk]), sv = __int_as_float(hd[kHdrSv]);
  const float qk = FP8 ? quant_recip(sk) : 0.f, qv = FP8 ? quant_recip(sv) : 0.f;
  const int p_lo = r0 + ch * kChunkPositions, p_hi = min(r1, p_lo + kChunkPositions);
  if (p_lo >= p_hi) return;
  const int b = hid / c.Hkv, h = hid % c.Hkv;
  const long long hi = head_index(c, in.layer, b, h);
  const long long in_stride = (long long)c.Hkv * c.D;
  const uint16_t* k_rows = in.k_in + ((long long)b * in.max_new * c.Hkv + h) * c.D;
  const uint16_t* v_rows = in.v_in + ((long long)b * in.max_new * c.Hkv + h) * c.D;
  const uint8_t* keep_rows = in.keep_in + (long long)b * in.max_new * c.Hkv + h;
  const uint8_t* rkeep = c.ring_keep + hi * c.Rpad;
  const int32_t* bt = c.block_table + hi * c.max_blocks;
  const int VPR = c.D / 8;
  unsigned sat = 0;
  // survivors of the chunk, in position order: ballot inside warps, scan of
  // the warp totals, 256 positions at a time
  if (tid == 0) s_total = 0;
  __syncthreads();
  for (int base = p_lo; base < p_hi; base += kAppendThreads) {
    const int p = base + tid;
    int bit = 0;
    if (p < p_hi)
      bit = p < n0 ? (rkeep[p % c.R] != 0) : (keep_rows[(long long)(p - n0) * c.Hkv] != 0);
    const unsigned ball = __ballot_sync(0xffffffffu, bit);
    const int in_warp = __popc(ball & ((1u << lane) - 1u));
    if (lane == 0) s_warp[warp] = __popc(ball);
    __syncthreads();
    int warp_off = s_total, round = 0;
    for (int i = 0; i < kWarps; ++i) {
      warp_off += (i < warp) ? s_warp[i] : 0;
      round += s_warp[i];
    }
    if (bit) s_src[warp_off + in_warp] = p;
    __syncthreads();
    if (tid == 0) s_total += round;
    __syncthreads();
  }
  const int total = s_total;
  const int first = len0 + aw.counts[(long long)hid * aw.max_chunks + ch];   // store row
  // copy: (survivor, vector) pairs over the CTA, four loads in flight per thread
  for (int i0 = tid; i0 < total * VPR; i0 += 4 * kAppendThreads) {
    uint4 xk[4], xv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kAppendThreads;
      if (i >= total * VPR) break;
      const int src = s_src[i / VPR], vec = i % VPR;
      if (src < n0) {   // from the ring: already in cache format
        const int slot = src % c.R;
        const uint8_t* ks = ring_k(c, hi) + (long long)slot * c.RB;
        const uint8_t* vs = ring_v(c, hi) + (long long)slot * c.RB;
        if constexpr (FP8) {
          const uint2 a = *reinterpret_cast<const uint2*>(ks + swz_byte(c.RB, false, slot, vec * 8));
          const uint2 bb = *reinterpret_cast<const uint2*>(vs + swz_byte(c.RB, true, slot, vec * 8));
          xk[u] = make_uint4(a.x, a.y, 0u, 0u);
          xv[u] = make_uint4(bb.x, bb.y, 0u, 0u);
        } else {
          xk[u] = *reinterpret_cast<const uint4*>(ks + swz_byte(c.RB, false, slot, vec * 16));
          xv[u] = *reinterpret_cast<const uint4*>(vs + swz_byte(c.RB, true, slot, vec * 16));
        }
      } else {          // straight from this call's input
        const long long t = src - n0;
        xk[u] = *reinterpret_cast<const uint4*>(k_rows + t * in_stride + vec * 8);
        xv[u] = *reinterpret_cast<const uint4*>(v_rows + t * in_stride + vec * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kAppendThreads;
      if (i >= total * VPR) break;
      const int sidx = i / VPR, vec = i % VPR;
      const int src = s_src[sidx];
      const int d = first + sidx;
      const long long blk = bt[d / kBlockSlots];
      const int row = d % kBlockSlots;
      uint8_t* kd = block_k(c, blk) + (long long)row * c.RB;
      uint8_t* vd = block_v(c, blk) + (long long)row * c.RB;
      if constexpr (FP8) {
        const uint2 ok =
            src < n0 ? make_uint2(xk[u].x, xk[u].y) : quantise8(xk[u], sk, qk, sat);
        const uint2 ov =
            src < n0 ? make_uint2(xv[u].x, xv[u].y) : quantise8(xv[u], sv, qv, sat);
        *reinterpret_cast<uint2*>(kd + swz_byte(c.RB, false, row, vec * 8)) = ok;
        *reinterpret_cast<uint2*>(vd + swz_byte(c.RB, true, row, vec * 8)) = ov;
      } else {
        *reinterpret_cast<uint4*>(kd + swz_byte(c.RB, false, row, vec * 16)) = xk[u];
        *reinterpret_cast<uint4*>(vd + swz_byte(c.RB, true, row, vec * 16)) = xv[u];
      }
      if (vec == 0) c.blk_pos[blk * kBlockSlots + row] = src;
    }
  }
  if constexpr (FP8) {
    for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(0xffffffffu, sat, off);
    if (lane == 0 && sat) atomicAdd(&c.ctr->saturations, (unsigned long long)sat);
  }
}

template <bool FP8>
__global__ void __launch_bounds__(kAppendThreads)
k_bulk_ring(CacheView c, AppendWork aw, BulkIn in) {
  pdl_wait();
  pdl_launch_dependents();
  const int hid = blockIdx.x, tid = threadIdx.x, lane = tid % 32;
  const int* hd = aw.hdr + (long long)hid * kHdrInts;
  if (hd[kHdrStatus] != kBulkGo) return;
  const int n0 = hd[kHdrN0], n1 = hd[kHdrN1], r1 = hd[kHdrR1];
  const float sk = __int_as_float(hd[kHdrSk]), sv = __int_as_float(hd[kHdrSv]);
  const float qk = FP8 ? quant_recip(sk) : 0.f, qv = FP8 ? quant_recip(sv) : 0.f;
  const int b = hid / c.Hkv, h = hid % c.Hkv;
  const long long hi = head_index(c, in.layer, b, h);
  const long long in_stride = (long long)c.Hkv * c.D;
  const uint16_t* k_rows = in.k_in + ((long long)b * in.max_new * c.Hkv + h) * c.D;
  const uint16_t* v_rows = in.v_in + ((long long)b * in.max_new * c.Hkv + h) * c.D;
  const uint8_t* keep_rows = in.keep_in + (long long)b * in.max_new * c.Hkv + h;
  uint8_t* rkeep = c.ring_keep + hi * c.Rpad;
  const int VPR = c.D / 8;
  unsigned sat = 0;
  // vectors of rows w0 .. n1-1, spread over the gridDim.y CTAs of the head;
  // each thread loads its (up to) 4 input vectors before any store
  const int w0 = r1 > n0 ? r1 : n0;
  const long long nvec = (long long)(n1 - w0) * VPR;
  const long long stride = (long long)gridDim.y * kAppendThreads;
  for (long long i0 = (long long)blockIdx.y * kAppendThreads + tid; i0 < nvec; i0 += 4 * stride) {
    uint4 xk[4], xv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long i = i0 + u * stride;
      if (i < nvec) {
        const long long t = w0 + i / VPR - n0;
        const int vec = (int)(i % VPR);
        xk[u] = *reinterpret_cast<const uint4*>(k_rows + t * in_stride + vec * 8);
        xv[u] = *reinterpret_cast<const uint4*>(v_rows + t * in_stride + vec * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long i = i0 + u * stride;
      if (i >= nvec) break;
      const int p = w0 + (int)(i / VPR), vec = (int)(i % VPR);
      const int slot = p % c.R;
      uint8_t* kd = ring_k(c, hi) + (long long)slot * c.RB;
      uint8_t* vd = ring_v(c, hi) + (long long)slot * c.RB;
      if constexpr (FP8) {
        *reinterpret_cast<uint2*>(kd + swz_byte(c.RB, false, slot, vec * 8)) =
            quantise8(xk[u], sk, qk, sat);
        *reinterpret_cast<uint2*>(vd + swz_byte(c.RB, true, slot, vec * 8)) =
            quantise8(xv[u], sv, qv, sat);
      } else {
        *reinterpret_cast<uint4*>(kd + swz_byte(c.RB, false, slot, vec * 16)) = xk[u];
        *reinterpret_cast<uint4*>(vd + swz_byte(c.RB, true, slot, vec * 16)) = xv[u];
      }
      if (vec == 0) rkeep[slot] = keep_rows[(p - n0) * c.Hkv] ? 1 : 0;
    }
  }
  if constexpr (FP8) {
    for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(0xffffffffu, sat, off);
    if (lane == 0 && sat) atomicAdd(&c.ctr->saturations, (unsigned long long)sat);
  }
}

constexpr int kSmallMax = 16;
constexpr int kSmallWarps = 8;

// Resolution, ring writes and length update of one (seq, kv head) for the
// warp-per-head paths: positions r0 .. r1-1 are resolved (survivors appended to
// the store in order), positions max(r1, n0) .. n1-1 go to the ring.
template <bool FP8>
__device__ void warp_resolve(const CacheView& c, long long hi, int lane, int n0, int r0,
                             int len0, int n1, int r1, float sk, float sv,
                             const uint16_t* k_rows, const uint16_t* v_rows,
                             const uint8_t* keep_rows, long long in_stride) {
  uint8_t* rkeep = c.ring_keep + hi * c.Rpad;
  const int VPR = c.D / 8;    // 16-byte input vectors per row
  const float qk = FP8 ? quant_recip(sk) : 0.f, qv = FP8 ? quant_recip(sv) : 0.f;
  auto keep_of = [&](int p) -> int {
    return p < n0 ? (rkeep[p % c.R] != 0) : (keep_rows[(long long)(p - n0) * c.Hkv] != 0);
  };
  // survivors of positions r0 .. r1-1, and their blocks
  int total = 0;
  for (int base = r0; base < r1; base += 32) {
    const int p = base + lane;
    total += __popc(__ballot_sync(0xffffffffu, p < r1 && keep_of(p)));
  }
  const int len1 = len0 + total;
  const int nb0 = (len0 + kBlockSlots - 1) / kBlockSlots;
  const int nb1 = (len1 + kBlockSlots - 1) / kBlockSlots;
  long long base_blk = 0;
  if (nb1 > nb0) {
    int fail = 0;
    if (lane == 0) {
      base_blk = take_blocks(c.ctr, (unsigned long long)(nb1 - nb0), c.num_blocks);
      if (base_blk < 0) {
        latch_error(c.ctr, FDMS_ERR_OUT_OF_BLOCKS);
        fail = 1;
      }
    }
    if (__shfl_sync(0xffffffffu, fail, 0)) return;
    base_blk = __shfl_sync(0xffffffffu, base_blk, 0);
  }
  int32_t* bt = c.block_table + hi * c.max_blocks;
  float* bts = c.bt_scale + hi * c.max_blocks * 2;
  for (int j = nb0 + lane; j < nb1; j += 32) {
    bt[j] = (int32_t)(base_blk + (j - nb0));
    bts[2 * j] = sk;
    bts[2 * j + 1] = sv;
  }
  const long long tail_blk = (len0 % kBlockSlots) ? bt[nb0 - 1] : 0;   // partly filled block
  __syncwarp();

  unsigned sat = 0;
  int written = 0;
  for (int base = r0; base < r1; base += 32) {
    const int p = base + lane;
    const unsigned ball = __ballot_sync(0xffffffffu, p < r1 && keep_of(p));
    const int cnt = __popc(ball);
    for (int i = lane; i < cnt * VPR; i += 32) {
      const int sidx = i / VPR, vec = i % VPR;
      const int src = base + (int)__fns(ball, 0, sidx + 1);
      const int d = len0 + written + sidx;
      const int j = d / kBlockSlots;
      const long long blk = j < nb0 ? tail_blk : base_blk + (j - nb0);
      const int row = d % kBlockSlots;
      uint8_t* kd = block_k(c, blk) + (long long)row * c.RB;
      uint8_t* vd = block_v(c, blk) + (long long)row * c.RB;
      if (src < n0) {
        const int slot = src % c.R;
        move_vec<FP8>(kd, row, ring_k(c, hi) + (long long)slot * c.RB, slot, vec, c.RB, false);
        move_vec<FP8>(vd, row, ring_v(c, hi) + (long long)slot * c.RB, slot, vec, c.RB, true);
      } else {
        const long long t = src - n0;
        put_input_vec<FP8>(kd, k_rows + t * in_stride, vec, sk, qk, sat, c.RB, false, row);
        put_input_vec<FP8>(vd, v_rows + t * in_stride, vec, sv, qv, sat, c.RB, true, row);
      }
      if (vec == 0) c.blk_pos[blk * kBlockSlots + row] = src;
    }
    written += cnt;
  }
  __syncwarp();   // ring slots read above may be overwritten below

  const int w0 = r1 > n0 ? r1 : n0;
  for (int i = lane; i < (n1 - w0) * VPR; i += 32) {
    const int p = w0 + i / VPR, vec = i % VPR;
    const long long t = p - n0;
    const int slot = p % c.R;
    put_input_vec<FP8>(ring_k(c, hi) + (long long)slot * c.RB, k_rows + t * in_stride, vec, sk,
                       qk, sat, c.RB, false, slot);
    put_input_vec<FP8>(ring_v(c, hi) + (long long)slot * c.RB, v_rows + t * in_stride, vec, sv,
                       qv, sat, c.RB, true, slot);
    if (vec == 0) rkeep[slot] = keep_rows[t * c.Hkv] ? 1 : 0;
  }
  if constexpr (FP8) {
    for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(0xffffffffu, sat, off);
    if (lane == 0 && sat) atomicAdd(&c.ctr->saturations, (unsigned long long)sat);
  }
  __syncwarp();
  if (lane == 0) {
    c.store_len[hi] = len1;
    c.tok_n[hi] = n1;
    c.tok_r[hi] = r1;
  }
}

// Decode-step path: one warp per (seq, kv head), for calls that bring at most
// kSmallMax tokens per sequence. Same semantics as the bulk path; the loads
// whose addresses are known are issued together, so a decode step costs about
// two dependent memory round trips.

template <bool FP8>
__global__ void __launch_bounds__(kSmallWarps * 32)
k_append_small(CacheView c, int layer, int batch, const int32_t* __restrict__ n_new, int max_new,
               const uint16_t* __restrict__ k_in, const uint16_t* __restrict__ v_in,
               const uint8_t* __restrict__ keep_in, const float* __restrict__ kv_scale) {
  pdl_wait();                 // the previous kernel's writes are visible from here on
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int hid = blockIdx.x * kSmallWarps + (threadIdx.x >> 5);
  if (hid >= batch * c.Hkv) return;
  const int b = hid / c.Hkv, h = hid % c.Hkv;
  const long long hi = head_index(c, layer, b, h);
  const long long in_stride = (long long)c.Hkv * c.D;   // elements between tokens
  const uint16_t* k_rows = k_in + ((long long)b * max_new * c.Hkv + h) * c.D;
  const uint16_t* v_rows = v_in + ((long long)b * max_new * c.Hkv + h) * c.D;
  const uint8_t* keep_rows = keep_in + (long long)b * max_new * c.Hkv + h;
  const int VPR = c.D / 8;    // 16-byte input vectors per row

  const int m = n_new[b];
  const int n0 = c.tok_n[hi], r0 = c.tok_r[hi], len0 = c.store_len[hi];
  if (m < 0 || m > max_new) {
    if (lane == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
    return;
  }
  if (m == 0) return;
  if ((long long)n0 + m > c.max_seq_len) {
    if (lane == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
    return;
  }
  const int n1 = n0 + m;
  const int r1 = (n1 - c.W - r0 >= c.P) ? n1 - c.W : r0;

  float sk = 1.0f, sv = 1.0f;
  if constexpr (FP8) {
    if (n0 == 0) {
      if (kv_scale) {
        sk = kv_scale[((long long)b * c.Hkv + h) * 2];
        sv = kv_scale[((long long)b * c.Hkv + h) * 2 + 1];
      } else {
        float ak = 0.f, av = 0.f;
        for (int i = lane; i < m * VPR; i += 32) {
          const long long row = i / VPR;
          const int vec = i % VPR;
          const uint4 xk = *reinterpret_cast<const uint4*>(k_rows + row * in_stride + vec * 8);
          const uint4 xv = *reinterpret_cast<const uint4*>(v_rows + row * in_stride + vec * 8);
          const uint32_t wk[4] = {xk.x, xk.y, xk.z, xk.w}, wv[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ak = fmaxf(ak, fmaxf(fabsf(bf16lo_to_f32(wk[j])), fabsf(bf16hi_to_f32(wk[j]))));
            av = fmaxf(av, fmaxf(fabsf(bf16lo_to_f32(wv[j])), fabsf(bf16hi_to_f32(wv[j]))));
          }
        }
        for (int off = 16; off > 0; off >>= 1) {
          ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, off));
          av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, off));
        }
        sk = __fdiv_rn(fmaxf(ak, 1.17549435e-38f), 448.0f);
        sv = __fdiv_rn(fmaxf(av, 1.17549435e-38f), 448.0f);
      }
      if (lane == 0) {
        c.head_scale[hi * 2] = sk;
        c.head_scale[hi * 2 + 1] = sv;
      }
    } else {
      sk = c.head_scale[hi * 2];
      sv = c.head_scale[hi * 2 + 1];
    }
  }

  warp_resolve<FP8>(c, hi, lane, n0, r0, len0, n1, r1, sk, sv, k_rows, v_rows, keep_rows,
                    in_stride);
}

// Decode steps proper: at most kStepVecs 16-byte input vectors per sequence
// (max_new * D / 8 <= 32), one warp per (seq, kv head). Same result as
// k_append_small; ordered for latency. A head's own state (lengths, FP8
// scales, ring keep bits and rows, block table) is written only by appends to
// its layer. When the host knows that the last append to this layer has
// finished by the time this grid starts (`state_early`), the state, and the
// ring rows of every position the call could resolve, are read before the
// wait, while the previous kernel still runs, and only the call's own inputs
// are read after it: a step costs one round trip to memory after the wait
// (two when the store needs a new block). Without `state_early` the same loads
// come after the wait, in two round trips. Resolutions larger than two
// vectors per lane take the general path.
constexpr int kStepVecs = 32;

template <bool FP8>
__global__ void __maxnreg__(128)   // room for the rows read early (the default target spills)
k_append_step(CacheView c, int layer, int batch, const int32_t* __restrict__ n_new, int max_new,
              const uint16_t* __restrict__ k_in, const uint16_t* __restrict__ v_in,
              const uint8_t* __restrict__ keep_in, const float* __restrict__ kv_scale,
              int state_early) {
  // The next kernel may start at once: it reads nothing this one writes
  // before its own dependency wait (the host keeps track of which kernels have
  // certainly finished when deciding what may be read early).
  pdl_launch_dependents();
  if (!state_early) pdl_wait();   // the previous kernel's writes are visible from here on
  const int lane = threadIdx.x & 31;
  const int hid = blockIdx.x * kSmallWarps + (threadIdx.x >> 5);
  if (hid >= batch * c.Hkv) {
    if (state_early) pdl_wait();
    return;
  }
  const int b = hid / c.Hkv, h = hid % c.Hkv;
  const long long hi = head_index(c, layer, b, h);
  const long long in_stride = (long long)c.Hkv * c.D;   // elements between tokens
  const uint16_t* k_rows = k_in + ((long long)b * max_new * c.Hkv + h) * c.D;
  const uint16_t* v_rows = v_in + ((long long)b * max_new * c.Hkv + h) * c.D;
  const uint8_t* keep_rows = keep_in + (long long)b * max_new * c.Hkv + h;
  uint8_t* rkeep = c.ring_keep + hi * c.Rpad;
  int32_t* bt = c.block_table + hi * c.max_blocks;
  const int VPR = c.D / 8;    // 16-byte input vectors per row
  constexpr unsigned kAll = 0xffffffffu;
  constexpr int EV = FP8 ? 8 : 16;   // bytes of one vector in the cache

  // ---- the head's state and the ring rows the call may resolve
  const int n0 = c.tok_n[hi], r0 = c.tok_r[hi], len0 = c.store_len[hi];
  float sk = 1.0f, sv = 1.0f, qk = 0.f, qv = 0.f;
  if constexpr (FP8) {
    sk = c.head_scale[hi * 2];
    sv = c.head_scale[hi * 2 + 1];
    qk = quant_recip(sk);
    qv = quant_recip(sv);
  }
  // positions resolved if the sequence brings max_new tokens: resolution is
  // monotone in the count, so these cover what any count up to max_new resolves
  const int nm = n0 + max_new;
  const int res_m = (nm - c.W - r0 >= c.P) ? nm - c.W - r0 : 0;
  const bool fast = res_m <= 32 && res_m * VPR <= 2 * 32;
  int kring = 0;
  uint4 rk[2], rv[2];
  long long tail_blk = 0;
#pragma unroll
  for (int j = 0; j < 2; ++j) rk[j] = rv[j] = make_uint4(0u, 0u, 0u, 0u);
  if (fast) {
    if (lane < res_m && r0 + lane < n0) kring = rkeep[(r0 + lane) % c.R] != 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int i = lane + 32 * j;
      if (i < res_m * VPR) {
        const int p = r0 + i / VPR, vec = i % VPR;
        if (p < n0) {
          const int slot = p % c.R;
          const uint8_t* ks = ring_k(c, hi) + (long long)slot * c.RB;
          const uint8_t* vs = ring_v(c, hi) + (long long)slot * c.RB;
          if constexpr (FP8) {
            const uint2 a =
                *reinterpret_cast<const uint2*>(ks + swz_byte(c.RB, false, slot, vec * EV));
            const uint2 bb =
                *reinterpret_cast<const uint2*>(vs + swz_byte(c.RB, true, slot, vec * EV));
            rk[j] = make_uint4(a.x, a.y, 0u, 0u);
            rv[j] = make_uint4(bb.x, bb.y, 0u, 0u);
          } else {
            rk[j] = *reinterpret_cast<const uint4*>(ks + swz_byte(c.RB, false, slot, vec * EV));
            rv[j] = *reinterpret_cast<const uint4*>(vs + swz_byte(c.RB, true, slot, vec * EV));
          }
        }
      }
    }
    if (len0 % kBlockSlots) tail_blk = bt[(len0 - 1) / kBlockSlots];   // partly filled block
  }
  if (state_early) pdl_wait();

  // ---- the call's inputs: count, rows (vector `lane`), keep bits
  const int m = n_new[b];
  uint4 xk = make_uint4(0u, 0u, 0u, 0u), xv = xk;
  if (lane < max_new * VPR) {
    const int t = lane / VPR, vec = lane % VPR;
    xk = *reinterpret_cast<const uint4*>(k_rows + t * in_stride + vec * 8);
    xv = *reinterpret_cast<const uint4*>(v_rows + t * in_stride + vec * 8);
  }
  const int knew = lane < max_new ? (keep_rows[(long long)lane * c.Hkv] != 0) : 0;
  if (m < 0 || m > max_new || (long long)n0 + m > c.max_seq_len) {
    if (lane == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
    return;
  }
  if (m == 0) return;
  const int n1 = n0 + m;
  const int r1 = (n1 - c.W - r0 >= c.P) ? n1 - c.W : r0;
  if constexpr (FP8) {
    if (n0 == 0) {   // a sequence's first append fixes its scales
      if (kv_scale) {
        sk = kv_scale[((long long)b * c.Hkv + h) * 2];
        sv = kv_scale[((long long)b * c.Hkv + h) * 2 + 1];
      } else {
        float ak = 0.f, av = 0.f;
        if (lane < m * VPR) {
          const uint32_t wk[4] = {xk.x, xk.y, xk.z, xk.w}, wv[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ak = fmaxf(ak, fmaxf(fabsf(bf16lo_to_f32(wk[j])), fabsf(bf16hi_to_f32(wk[j]))));
            av = fmaxf(av, fmaxf(fabsf(bf16lo_to_f32(wv[j])), fabsf(bf16hi_to_f32(wv[j]))));
          }
        }
        for (int off = 16; off > 0; off >>= 1) {
          ak = fmaxf(ak, __shfl_xor_sync(kAll, ak, off));
          av = fmaxf(av, __shfl_xor_sync(kAll, av, off));
        }
        sk = __fdiv_rn(fmaxf(ak, 1.17549435e-38f), 448.0f);
        sv = __fdiv_rn(fmaxf(av, 1.17549435e-38f), 448.0f);
      }
      if (lane == 0) {
        c.head_scale[hi * 2] = sk;
        c.head_scale[hi * 2 + 1] = sv;
      }
      qk = quant_recip(sk);
      qv = quant_recip(sv);
    }
  }
  const int nres = r1 - r0;   // <= res_m
  if (!fast) {
    warp_resolve<FP8>(c, hi, lane, n0, r0, len0, n1, r1, sk, sv, k_rows, v_rows, keep_rows,
                      in_stride);
    return;
  }

  // keep bits of the resolved positions: ring bits read above, the call's own
  const int p_l = r0 + lane;
  const int knew_p = __shfl_sync(kAll, knew, (p_l - n0) & 31);
  const int kp = lane < nres ? (p_l < n0 ? kring : knew_p) : 0;
  const unsigned ball = __ballot_sync(kAll, kp != 0);
  const int len1 = len0 + __popc(ball);
  const int nb0 = (len0 + kBlockSlots - 1) / kBlockSlots;
  const int nb1 = (len1 + kBlockSlots - 1) / kBlockSlots;
  long long base_blk = 0;
  if (nb1 > nb0) {   // new store blocks for this call, reserved at once
    int fail = 0;
    if (lane == 0) {
      base_blk = take_blocks(c.ctr, (unsigned long long)(nb1 - nb0), c.num_blocks);
      if (base_blk < 0) {
        latch_error(c.ctr, FDMS_ERR_OUT_OF_BLOCKS);
        fail = 1;
      }
    }
    if (__shfl_sync(kAll, fail, 0)) return;
    base_blk = __shfl_sync(kAll, base_blk, 0);
    float* bts = c.bt_scale + hi * c.max_blocks * 2;
    for (int j = nb0 + lane; j < nb1; j += 32) {
      bt[j] = (int32_t)(base_blk + (j - nb0));
      bts[2 * j] = sk;
      bts[2 * j + 1] = sv;
    }
  }

  // ---- writes: survivors to the store, in position order
  unsigned sat = 0;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int i = lane + 32 * j;
    if (i >= nres * VPR) continue;
    const int ri = i / VPR, vec = i % VPR;
    if (!((ball >> ri) & 1u)) continue;
    const int d = len0 + __popc(ball & ((1u << ri) - 1u));
    const int jb = d / kBlockSlots, row = d % kBlockSlots;
    const long long blk = jb < nb0 ? tail_blk : base_blk + (jb - nb0);
    uint8_t* kd = block_k(c, blk) + (long long)row * c.RB;
    uint8_t* vd = block_v(c, blk) + (long long)row * c.RB;
    const int p = r0 + ri;
    if (p < n0) {
      if constexpr (FP8) {
        *reinterpret_cast<uint2*>(kd + swz_byte(c.RB, false, row, vec * EV)) =
            make_uint2(rk[j].x, rk[j].y);
        *reinterpret_cast<uint2*>(vd + swz_byte(c.RB, true, row, vec * EV)) =
            make_uint2(rv[j].x, rv[j].y);
      } else {
        *reinterpret_cast<uint4*>(kd + swz_byte(c.RB, false, row, vec * EV)) = rk[j];
        *reinterpret_cast<uint4*>(vd + swz_byte(c.RB, true, row, vec * EV)) = rv[j];
      }
    } else {   // a token of this call resolved at once (window shorter than the call)
      const long long t = p - n0;
      put_input_vec<FP8>(kd, k_rows + t * in_stride, vec, sk, qk, sat, c.RB, false, row);
      put_input_vec<FP8>(vd, v_rows + t * in_stride, vec, sv, qv, sat, c.RB, true, row);
    }
    if (vec == 0) c.blk_pos[blk * kBlockSlots + row] = p;
  }

  // ---- the call's unresolved tokens to the ring; a new token can take the
  // ring slot of a position resolved above, whose row was read in round trip 2
  __syncwarp();
  const int w0 = r1 > n0 ? r1 : n0;
  {
    const int t = lane / VPR, vec = lane % VPR, p = n0 + t;
    const int keep_t = __shfl_sync(kAll, knew, t & 31);
    if (lane < m * VPR && p >= w0) {
      const int slot = p % c.R;
      uint8_t* kd = ring_k(c, hi) + (long long)slot * c.RB;
      uint8_t* vd = ring_v(c, hi) + (long long)slot * c.RB;
      if constexpr (FP8) {
        *reinterpret_cast<uint2*>(kd + swz_byte(c.RB, false, slot, vec * EV)) =
            quantise8(xk, sk, qk, sat);
        *reinterpret_cast<uint2*>(vd + swz_byte(c.RB, true, slot, vec * EV)) =
            quantise8(xv, sv, qv, sat);
      } else {
        *reinterpret_cast<uint4*>(kd + swz_byte(c.RB, false, slot, vec * EV)) = xk;
        *reinterpret_cast<uint4*>(vd + swz_byte(c.RB, true, slot, vec * EV)) = xv;
      }
      if (vec == 0) rkeep[slot] = keep_t ? 1 : 0;
    }
  }
  if constexpr (FP8) {
    for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(kAll, sat, off);
    if (lane == 0 && sat) atomicAdd(&c.ctr->saturations, (unsigned long long)sat);
  }
  __syncwarp();
  if (lane == 0) {
    c.store_len[hi] = len1;
    c.tok_n[hi] = n1;
    c.tok_r[hi] = r1;
  }
}


// ===================================================== per-block FP8 append
// FDMS_KV_FP8_E4M3_BLOCK: survivors go, in order, to the head's bf16 staging
// block; when its 64th row is written the block is sealed: one pool block
// (taken from the bump allocator for all of the call's seals at once, before
// any write, so a head that does not fit is left unchanged), K and V scales
// max(amax over the 64 rows, 2^-126) / 448, the rows quantised into it with the
// same correctly rounded quotient as the other FP8 paths. New tokens that stay
// unresolved go to the ring as bf16. A warp per head, any call size (the
// survivors of a 32-position chunk cross at most one block boundary).

// 16-byte bf16 vector `vec` of row `row` in a bf16 page of `rb`-byte rows
__device__ __forceinline__ uint4* bf16_vec(uint8_t* page, int rb, bool is_v, int row, int vec) {
  return reinterpret_cast<uint4*>(page + (long long)row * rb + swz_byte(rb, is_v, row, vec * 16));
}

__device__ __forceinline__ float amax8(uint4 x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  float a = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    a = fmaxf(a, fmaxf(fabsf(bf16lo_to_f32(w[j])), fabsf(bf16hi_to_f32(w[j]))));
  return a;
}

// Seal the staging block of head hi as store block jb in pool block blk.
__device__ void seal_block(const CacheView& c, long long hi, int jb, long long blk, int lane,
                           unsigned& sat) {
  const int VPR = c.D / 8, SRB = 2 * c.D;
  uint8_t* sk = stage_k(c, hi);
  uint8_t* sv = stage_v(c, hi);
  float ak = 0.f, av = 0.f;
  for (int i = lane; i < kBlockSlots * VPR; i += 32) {
    const int row = i / VPR, vec = i % VPR;
    ak = fmaxf(ak, amax8(*bf16_vec(sk, SRB, false, row, vec)));
    av = fmaxf(av, amax8(*bf16_vec(sv, SRB, true, row, vec)));
  }
  for (int off = 16; off > 0; off >>= 1) {
    ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, off));
    av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, off));
  }
  const float sck = __fdiv_rn(fmaxf(ak, 1.17549435e-38f), 448.0f);
  const float scv = __fdiv_rn(fmaxf(av, 1.17549435e-38f), 448.0f);
  const float qk = quant_recip(sck), qv = quant_recip(scv);
  uint8_t* dk = block_k(c, blk);
  uint8_t* dv = block_v(c, blk);
  for (int i = lane; i < kBlockSlots * VPR; i += 32) {
    const int row = i / VPR, vec = i % VPR;
    *reinterpret_cast<uint2*>(dk + (long long)row * c.RB + swz_byte(c.RB, false, row, vec * 8)) =
        quantise8(*bf16_vec(sk, SRB, false, row, vec), sck, qk, sat);
    *reinterpret_cast<uint2*>(dv + (long long)row * c.RB + swz_byte(c.RB, true, row, vec * 8)) =
        quantise8(*bf16_vec(sv, SRB, true, row, vec), scv, qv, sat);
  }
  for (int row = lane; row < kBlockSlots; row += 32)
    c.blk_pos[blk * kBlockSlots + row] = c.stage_pos[hi * kBlockSlots + row];
  if (lane == 0) {
    c.block_table[hi * c.max_blocks + jb] = (int32_t)blk;
    c.bt_scale[(hi * c.max_blocks + jb) * 2] = sck;
    c.bt_scale[(hi * c.max_blocks + jb) * 2 + 1] = scv;
  }
}

__global__ void __launch_bounds__(kSmallWarps * 32)
k_append_block(CacheView c, int layer, int batch, const int32_t* __restrict__ n_new,
               int max_new, const uint16_t* __restrict__ k_in, const uint16_t* __restrict__ v_in,
               const uint8_t* __restrict__ keep_in) {
  pdl_wait();                 // the previous kernel's writes are visible from here on
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int hid = blockIdx.x * kSmallWarps + (threadIdx.x >> 5);
  if (hid >= batch * c.Hkv) return;
  const int b = hid / c.Hkv, h = hid % c.Hkv;
  const long long hi = head_index(c, layer, b, h);
  const long long in_stride = (long long)c.Hkv * c.D;   // elements between tokens
  const uint16_t* k_rows = k_in + ((long long)b * max_new * c.Hkv + h) * c.D;
  const uint16_t* v_rows = v_in + ((long long)b * max_new * c.Hkv + h) * c.D;
  const uint8_t* keep_rows = keep_in + (long long)b * max_new * c.Hkv + h;
  uint8_t* rkeep = c.ring_keep + hi * c.Rpad;
  const int VPR = c.D / 8, SRB = 2 * c.D;
  constexpr unsigned kAll = 0xffffffffu;

  const int m = n_new[b];
  const int n0 = c.tok_n[hi], r0 = c.tok_r[hi], len0 = c.store_len[hi];
  if (m < 0 || m > max_new || (long long)n0 + m > c.max_seq_len) {
    if (lane == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
    return;
  }
  if (m == 0) return;
  const int n1 = n0 + m;
  const int r1 = (n1 - c.W - r0 >= c.P) ? n1 - c.W : r0;
  auto keep_of = [&](int p) -> int {
    return p < n0 ? (rkeep[p % c.R] != 0) : (keep_rows[(long long)(p - n0) * c.Hkv] != 0);
  };

  // survivors, and the pool blocks the call seals (one bump, before any write)
  int total = 0;
  for (int base = r0; base < r1; base += 32) {
    const int p = base + lane;
    total += __popc(__ballot_sync(kAll, p < r1 && keep_of(p)));
  }
  const int len1 = len0 + total;
  const int nseal = len1 / kBlockSlots - len0 / kBlockSlots;
  long long base_blk = 0;
  if (nseal > 0) {
    int fail = 0;
    if (lane == 0) {
      const long long base = take_blocks(c.ctr, (unsigned long long)nseal, c.num_blocks);
      if (base < 0) {
        latch_error(c.ctr, FDMS_ERR_OUT_OF_BLOCKS);
        fail = 1;
      } else {
        base_blk = base;
      }
    }
    if (__shfl_sync(kAll, fail, 0)) return;
    base_blk = __shfl_sync(kAll, base_blk, 0);
  }

  // survivors to staging rows, in store order, sealing each block that fills
  unsigned sat = 0;
  uint8_t* sk = stage_k(c, hi);
  uint8_t* sv = stage_v(c, hi);
  int len = len0;
  auto stage_rows = [&](unsigned ball, int base, int k0, int k1, int d0) {
    // ranks k0 .. k1-1 of the chunk's survivors to store indices d0 + (rank - k0)
    for (int i = lane; i < (k1 - k0) * VPR; i += 32) {
      const int rank = k0 + i / VPR, vec = i % VPR;
      const int src = base + (int)__fns(ball, 0, rank + 1);
      const int row = (d0 + rank - k0) % kBlockSlots;
      uint4 xk, xv;
      if (src < n0) {
        const int slot = src % c.R;
        xk = *bf16_vec(ring_k(c, hi), SRB, false, slot, vec);
        xv = *bf16_vec(ring_v(c, hi), SRB, true, slot, vec);
      } else {
        const long long t = src - n0;
        xk = *reinterpret_cast<const uint4*>(k_rows + t * in_stride + vec * 8);
        xv = *reinterpret_cast<const uint4*>(v_rows + t * in_stride + vec * 8);
      }
      *bf16_vec(sk, SRB, false, row, vec) = xk;
      *bf16_vec(sv, SRB, true, row, vec) = xv;
      if (vec == 0) c.stage_pos[hi * kBlockSlots + row] = src;
    }
  };
  for (int base = r0; base < r1; base += 32) {
    const int p = base + lane;
    const unsigned ball = __ballot_sync(kAll, p < r1 && keep_of(p));
    const int cnt = __popc(ball);
    if (cnt == 0) continue;
    const int first = min(cnt, kBlockSlots - len % kBlockSlots);   // fills the open block
    stage_rows(ball, base, 0, first, len);
    len += first;
    if (len % kBlockSlots == 0) {
      __syncwarp();
      const int jb = len / kBlockSlots - 1;
      seal_block(c, hi, jb, base_blk + (jb - len0 / kBlockSlots), lane, sat);
      __syncwarp();   // the staging rows are read before the next ones are written
    }
    if (cnt > first) {
      stage_rows(ball, base, first, cnt, len);
      len += cnt - first;
    }
  }
  __syncwarp();   // ring slots read above may be overwritten below

  // the call's unresolved tokens to the ring, in bf16
  const int w0 = r1 > n0 ? r1 : n0;
  for (int i = lane; i < (n1 - w0) * VPR; i += 32) {
    const int p = w0 + i / VPR, vec = i % VPR;
    const long long t = p - n0;
    const int slot = p % c.R;
    *bf16_vec(ring_k(c, hi), SRB, false, slot, vec) =
        *reinterpret_cast<const uint4*>(k_rows + t * in_stride + vec * 8);
    *bf16_vec(ring_v(c, hi), SRB, true, slot, vec) =
        *reinterpret_cast<const uint4*>(v_rows + t * in_stride + vec * 8);
    if (vec == 0) rkeep[slot] = keep_rows[t * c.Hkv] ? 1 : 0;
  }
  for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(kAll, sat, off);
  if (lane == 0 && sat) atomicAdd(&c.ctr->saturations, (unsigned long long)sat);
  __syncwarp();
  if (lane == 0) {
    c.store_len[hi] = len1;
    c.tok_n[hi] = n1;
    c.tok_r[hi] = r1;
  }
}


// The same append for calls of many tokens (prefill): a CTA per (seq, kv head),
// its warps sharing the work that the warp version does in sequence.
//   1. each 32-position chunk of the positions resolved now: its survivors'
//      ballot (shared memory), then a scan of the chunk counts over the CTA;
//   2. the blocks this call seals, one warp each: its 64 rows are the staged
//      rows of the open block (store indices below len0) and the survivors of
//      ranks 0 .. (found by a search over the chunk prefix and the chunk's
//      ballot); the K and V maxima over the rows, then the rows quantised;
//   3. (after 2 has read the staging rows) the survivors past the last sealed
//      block to the staging block;
//   4. (after every ring row has been read) the unresolved tokens to the ring.
// Same arithmetic as seal_block: the result is bit-identical.
constexpr int kBlockCtaThreads = 256;
constexpr int kBlockCtaWarps = kBlockCtaThreads / 32;
constexpr int kBlockCtaMinTokens = 64;   // calls with at least this many tokens per sequence

inline size_t block_cta_smem(int max_new, const CacheView& c) {
  const long long nch = ((long long)max_new + c.W + c.P + 31) / 32 + 2;
  return (size_t)nch * 2 * sizeof(uint32_t);
}

__global__ void __launch_bounds__(kBlockCtaThreads)
k_append_block_cta(CacheView c, int layer, int batch, const int32_t* __restrict__ n_new,
                   int max_new, const uint16_t* __restrict__ k_in,
                   const uint16_t* __restrict__ v_in, const uint8_t* __restrict__ keep_in) {
  pdl_wait();                 // the previous kernel's writes are visible from here on
  pdl_launch_dependents();
  extern __shared__ uint32_t s_chunk[];   // [nch] survivor ballots, then [nch] prefixes
  __shared__ long long s_base;
  __shared__ int s_fail;
  __shared__ unsigned s_sat;
  __shared__ int s_row[kBlockCtaWarps][kBlockSlots];   // a block's rows: position, or -1 - row
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hid = blockIdx.x;
  if (hid >= batch * c.Hkv) return;
  const int b = hid / c.Hkv, h = hid % c.Hkv;
  const long long hi = head_index(c, layer, b, h);
  const long long in_stride = (long long)c.Hkv * c.D;   // elements between tokens
  const uint16_t* k_rows = k_in + ((long long)b * max_new * c.Hkv + h) * c.D;
  const uint16_t* v_rows = v_in + ((long long)b * max_new * c.Hkv + h) * c.D;
  const uint8_t* keep_rows = keep_in + (long long)b * max_new * c.Hkv + h;
  uint8_t* rkeep = c.ring_keep + hi * c.Rpad;
  const int VPR = c.D / 8, SRB = 2 * c.D;
  constexpr unsigned kAll = 0xffffffffu;

  const int m = n_new[b];
  const int n0 = c.tok_n[hi], r0 = c.tok_r[hi], len0 = c.store_len[hi];
  if (m < 0 || m > max_new || (long long)n0 + m > c.max_seq_len) {
    if (tid == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
    return;
  }
  if (m == 0) return;
  const int n1 = n0 + m;
  const int r1 = (n1 - c.W - r0 >= c.P) ? n1 - c.W : r0;
  const int nch = (r1 - r0 + 31) / 32;
  uint32_t* s_ball = s_chunk;
  uint32_t* s_pre = s_chunk + nch + 1;   // exclusive prefix of the chunk counts; [nch] = total
  auto keep_of = [&](int p) -> int {
    return p < n0 ? (rkeep[p % c.R] != 0) : (keep_rows[(long long)(p - n0) * c.Hkv] != 0);
  };

  // ---- 1. ballots and their prefix
  for (int ch = warp; ch < nch; ch += kBlockCtaWarps) {
    const int p = r0 + ch * 32 + lane;
    const unsigned ball = __ballot_sync(kAll, p < r1 && keep_of(p));
    if (lane == 0) s_ball[ch] = ball;
  }
  if (tid == 0) {
    s_fail = 0;
    s_sat = 0;
  }
  __syncthreads();
  if (warp == 0) {   // one warp scans: each lane a contiguous run of chunks
    const int per = (nch + 31) / 32;
    const int c0 = min(nch, lane * per), c1 = min(nch, c0 + per);
    unsigned run = 0;
    for (int ch = c0; ch < c1; ++ch) run += __popc(s_ball[ch]);
    unsigned inc = run;
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned y = __shfl_up_sync(kAll, inc, off);
      if (lane >= off) inc += y;
    }
    unsigned acc = inc - run;
    for (int ch = c0; ch < c1; ++ch) {
      s_pre[ch] = acc;
      acc += __popc(s_ball[ch]);
    }
    if (lane == 31) s_pre[nch] = inc;
  }
  __syncthreads();
  const int total = (int)s_pre[nch];
  const int len1 = len0 + total;
  const int jb0 = len0 / kBlockSlots, jb1 = len1 / kBlockSlots;   // blocks sealed: [jb0, jb1)
  if (tid == 0 && jb1 > jb0) {
    const long long base = take_blocks(c.ctr, (unsigned long long)(jb1 - jb0), c.num_blocks);
    if (base < 0) {
      latch_error(c.ctr, FDMS_ERR_OUT_OF_BLOCKS);
      s_fail = 1;
    }
    s_base = base;
  }
  __syncthreads();
  if (s_fail) return;
  const long long base_blk = s_base;

  // source position of survivor rank q (0 .. total-1): the chunk whose prefix
  // holds it (binary search), then the rank inside the chunk's ballot
  auto src_of = [&](int q) -> int {
    int lo = 0, hi_c = nch - 1;
    while (lo < hi_c) {
      const int mid = (lo + hi_c + 1) >> 1;
      if ((int)s_pre[mid] <= q) lo = mid;
      else hi_c = mid - 1;
    }
    return r0 + lo * 32 + (int)__fns(s_ball[lo], 0, q - (int)s_pre[lo] + 1);
  };
  // where store index d (>= 64 * jb0) comes from: the staged row (-1 - row)
  // or survivor d - len0's position; found once per row, by one lane
  uint8_t* sk = stage_k(c, hi);
  uint8_t* sv = stage_v(c, hi);
  auto row_src = [&](int d) -> int { return d < len0 ? -1 - d % kBlockSlots : src_of(d - len0); };
  // bf16 row vector `vec` of a row found by row_src, and the row's position
  auto row_vec = [&](int src, int vec, uint4& xk, uint4& xv, int& pos) {
    if (src < 0) {
      const int row = -1 - src;
      xk = *bf16_vec(sk, SRB, false, row, vec);
      xv = *bf16_vec(sv, SRB, true, row, vec);
      pos = c.stage_pos[hi * kBlockSlots + row];
    } else {
      pos = src;
      if (src < n0) {
        const int slot = src % c.R;
        xk = *bf16_vec(ring_k(c, hi), SRB, false, slot, vec);
        xv = *bf16_vec(ring_v(c, hi), SRB, true, slot, vec);
      } else {
        const long long t = src - n0;
        xk = *reinterpret_cast<const uint4*>(k_rows + t * in_stride + vec * 8);
        xv = *reinterpret_cast<const uint4*>(v_rows + t * in_stride + vec * 8);
      }
    }
  };
  int* rows_w = s_row[warp];

  // ---- 2. the sealed blocks, one warp each
  unsigned sat = 0;
  for (int jb = jb0 + warp; jb < jb1; jb += kBlockCtaWarps) {
    for (int row = lane; row < kBlockSlots; row += 32) rows_w[row] = row_src(jb * kBlockSlots + row);
    __syncwarp();
    float ak = 0.f, av = 0.f;
    for (int i = lane; i < kBlockSlots * VPR; i += 32) {
      const int row = i / VPR, vec = i % VPR;
      uint4 xk, xv;
      int pos;
      row_vec(rows_w[row], vec, xk, xv, pos);
      ak = fmaxf(ak, amax8(xk));
      av = fmaxf(av, amax8(xv));
    }
    for (int off = 16; off > 0; off >>= 1) {
      ak = fmaxf(ak, __shfl_xor_sync(kAll, ak, off));
      av = fmaxf(av, __shfl_xor_sync(kAll, av, off));
    }
    const float sck = __fdiv_rn(fmaxf(ak, 1.17549435e-38f), 448.0f);
    const float scv = __fdiv_rn(fmaxf(av, 1.17549435e-38f), 448.0f);
    const float qk = quant_recip(sck), qv = quant_recip(scv);
    const long long blk = base_blk + (jb - jb0);
    uint8_t* dk = block_k(c, blk);
    uint8_t* dv = block_v(c, blk);
    for (int i = lane; i < kBlockSlots * VPR; i += 32) {
      const int row = i / VPR, vec = i % VPR;
      uint4 xk, xv;
      int pos;
      row_vec(rows_w[row], vec, xk, xv, pos);
      *reinterpret_cast<uint2*>(dk + (long long)row * c.RB + swz_byte(c.RB, false, row, vec * 8)) =
          quantise8(xk, sck, qk, sat);
      *reinterpret_cast<uint2*>(dv + (long long)row * c.RB + swz_byte(c.RB, true, row, vec * 8)) =
          quantise8(xv, scv, qv, sat);
      if (vec == 0) c.blk_pos[blk * kBlockSlots + row] = pos;
    }
    if (lane == 0) {
      c.block_table[hi * c.max_blocks + jb] = (int32_t)blk;
      c.bt_scale[(hi * c.max_blocks + jb) * 2] = sck;
      c.bt_scale[(hi * c.max_blocks + jb) * 2 + 1] = scv;
    }
    __syncwarp();   // rows_w is read before the next block's rows are written
  }
  __syncthreads();   // the staged rows of the sealed block are read

  // ---- 3. the survivors past the last sealed block to the staging block
  const int d_lo = max(len0, jb1 * kBlockSlots);   // (fewer than 64 rows)
  int* rows_t = s_row[0];
  for (int k = tid; k < len1 - d_lo; k += kBlockCtaThreads) rows_t[k] = row_src(d_lo + k);
  __syncthreads();
  for (int i = tid; i < (len1 - d_lo) * VPR; i += kBlockCtaThreads) {
    const int d = d_lo + i / VPR, vec = i % VPR;
    uint4 xk, xv;
    int pos;
    row_vec(rows_t[d - d_lo], vec, xk, xv, pos);
    const int row = d % kBlockSlots;
    *bf16_vec(sk, SRB, false, row, vec) = xk;
    *bf16_vec(sv, SRB, true, row, vec) = xv;
    if (vec == 0) c.stage_pos[hi * kBlockSlots + row] = pos;
  }
  __syncthreads();   // ring slots read above may be overwritten below

  // ---- 4. the call's unresolved tokens to the ring, in bf16
  const int w0 = r1 > n0 ? r1 : n0;
  for (int i = tid; i < (n1 - w0) * VPR; i += kBlockCtaThreads) {
    const int p = w0 + i / VPR, vec = i % VPR;
    const long long t = p - n0;
    const int slot = p % c.R;
    *bf16_vec(ring_k(c, hi), SRB, false, slot, vec) =
        *reinterpret_cast<const uint4*>(k_rows + t * in_stride + vec * 8);
    *bf16_vec(ring_v(c, hi), SRB, true, slot, vec) =
        *reinterpret_cast<const uint4*>(v_rows + t * in_stride + vec * 8);
    if (vec == 0) rkeep[slot] = keep_rows[t * c.Hkv] ? 1 : 0;
  }
  for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(kAll, sat, off);
  if (lane == 0 && sat) atomicAdd(&s_sat, sat);
  __syncthreads();
  if (tid == 0) {
    if (s_sat) atomicAdd(&c.ctr->saturations, (unsigned long long)s_sat);
    c.store_len[hi] = len1;
    c.tok_n[hi] = n1;
    c.tok_r[hi] = r1;
  }
}

}  // namespace
}  // namespace fdms

using namespace fdms;

fdms_status fdms_launch_append(fdms_cache* cache, int layer, int batch, const int32_t* n_new,
                               int max_new, const void* k, const void* v, const uint8_t* keep,
                               const float* kv_scale, cudaStream_t s) {
  const CacheView& c = cache->view;
  const uint16_t* kk = static_cast<const uint16_t*>(k);
  const uint16_t* vv = static_cast<const uint16_t*>(v);
  const float* sc = c.fp8 && !c.blk ? kv_scale : nullptr;
  // this layer's state may be read before the dependency wait when its last
  // writer (the last append to the layer) has certainly finished
  const int early = fdms_log_finished(cache, cache->append_at[layer]) ? 1 : 0;
  long long last = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (c.blk && max_new >= kBlockCtaMinTokens) {   // per-block FP8, many tokens: a CTA per head
    cfg.gridDim = dim3((unsigned)(batch * c.Hkv));
    cfg.blockDim = dim3(kBlockCtaThreads);
    cfg.dynamicSmemBytes = block_cta_smem(max_new, c);
    if (cfg.dynamicSmemBytes > 48 * 1024) return FDMS_ERR_INVALID_ARG;
    e = cudaLaunchKernelEx(&cfg, k_append_block_cta, c, layer, batch, n_new, max_new, kk, vv,
                           keep);
    last = fdms_log_launch(cache, true);
  } else if (c.blk) {   // per-block FP8, a few tokens: a warp per head
    cfg.gridDim = dim3((unsigned)((batch * c.Hkv + kSmallWarps - 1) / kSmallWarps));
    cfg.blockDim = dim3(kSmallWarps * 32);
    e = cudaLaunchKernelEx(&cfg, k_append_block, c, layer, batch, n_new, max_new, kk, vv, keep);
    last = fdms_log_launch(cache, true);
  } else if (max_new * (c.D / 8) <= kStepVecs) {
    cfg.gridDim = dim3((unsigned)((batch * c.Hkv + kSmallWarps - 1) / kSmallWarps));
    cfg.blockDim = dim3(kSmallWarps * 32);
    e = c.fp8 ? cudaLaunchKernelEx(&cfg, k_append_step<true>, c, layer, batch, n_new, max_new,
                                   kk, vv, keep, sc, early)
              : cudaLaunchKernelEx(&cfg, k_append_step<false>, c, layer, batch, n_new, max_new,
                                   kk, vv, keep, sc, early);
    last = fdms_log_launch(cache, false);   // lets its successor start at once
  } else if (max_new <= kSmallMax) {
    cfg.gridDim = dim3((unsigned)((batch * c.Hkv + kSmallWarps - 1) / kSmallWarps));
    cfg.blockDim = dim3(kSmallWarps * 32);
    e = c.fp8 ? cudaLaunchKernelEx(&cfg, k_append_small<true>, c, layer, batch, n_new, max_new,
                                   kk, vv, keep, sc)
              : cudaLaunchKernelEx(&cfg, k_append_small<false>, c, layer, batch, n_new, max_new,
                                   kk, vv, keep, sc);
    last = fdms_log_launch(cache, true);
  } else {
    const AppendWork& aw = cache->awork;
    const BulkIn in{n_new, kk, vv, keep, sc, batch, max_new, layer};
    const long long span = (long long)max_new + c.W + c.P;   // bound on positions resolved
    const int nch = (int)((span + kChunkPositions - 1) / kChunkPositions);
    if (nch > aw.max_chunks) return FDMS_ERR_INVALID_ARG;
    const unsigned heads = (unsigned)(batch * c.Hkv);
    cfg.gridDim = dim3(heads, (unsigned)nch);
    cfg.blockDim = dim3(kAppendThreads);
    e = c.fp8 ? cudaLaunchKernelEx(&cfg, k_bulk_count<true>, c, aw, in)
              : cudaLaunchKernelEx(&cfg, k_bulk_count<false>, c, aw, in);
    last = fdms_log_launch(cache, true);
    if (e == cudaSuccess) {
      cfg.gridDim = dim3(1);
      cfg.blockDim = dim3(kAllocThreads);
      cfg.dynamicSmemBytes = bulk_alloc_smem((int)heads);
      e = c.fp8 ? cudaLaunchKernelEx(&cfg, k_bulk_alloc<true>, c, aw, in, nch, (int)heads)
                : cudaLaunchKernelEx(&cfg, k_bulk_alloc<false>, c, aw, in, nch, (int)heads);
      last = fdms_log_launch(cache, true);
    }
    if (e == cudaSuccess) {
      cfg.gridDim = dim3(heads, (unsigned)nch);
      cfg.blockDim = dim3(kAppendThreads);
      cfg.dynamicSmemBytes = 0;
      e = c.fp8 ? cudaLaunchKernelEx(&cfg, k_bulk_write<true>, c, aw, in)
                : cudaLaunchKernelEx(&cfg, k_bulk_write<false>, c, aw, in);
      last = fdms_log_launch(cache, true);
    }
    if (e == cudaSuccess) {   // ring rows: at most W + P - 1 + max_new per head
      const long long rvec = (long long)min((long long)max_new, (long long)c.W + c.P) * (c.D / 8);
      const int ry = (int)std::min<long long>(16, (rvec + 4LL * kAppendThreads - 1) /
                                                    (4LL * kAppendThreads));
      cfg.gridDim = dim3(heads, (unsigned)std::max(1, ry));
      e = c.fp8 ? cudaLaunchKernelEx(&cfg, k_bulk_ring<true>, c, aw, in)
                : cudaLaunchKernelEx(&cfg, k_bulk_ring<false>, c, aw, in);
      last = fdms_log_launch(cache, true);
    }
  }
  if (last > 0) {
    cache->append_at[layer] = last;
    cache->tokens_since[layer] += max_new;
  }
  return e == cudaSuccess ? FDMS_OK : FDMS_ERR_CUDA;
}

fdms_status fdms_append_setup(fdms_cache* cache) {
  const CacheView& c = cache->view;
  AppendWork& aw = cache->awork;
  const long long span = (long long)c.max_seq_len + c.W + c.P;
  aw.max_chunks = (int)((span + kChunkPositions - 1) / kChunkPositions);
  const size_t heads = (size_t)c.Bmax * c.Hkv;
  void* p = nullptr;
  auto take = [&](size_t bytes) -> void* {
    if (cudaMalloc(&p, bytes) != cudaSuccess || !fdms_track(cache, p, bytes)) return nullptr;
    if (cudaMemset(p, 0, bytes) != cudaSuccess) return nullptr;
    return p;
  };
  aw.counts = static_cast<int*>(take(heads * aw.max_chunks * sizeof(int)));
  aw.hdr = static_cast<int*>(take(heads * kHdrInts * sizeof(int)));
  aw.amax = static_cast<unsigned*>(take(heads * 2 * sizeof(unsigned)));
  const int smem = (int)bulk_alloc_smem((int)heads);
  if (cudaFuncSetAttribute(k_bulk_alloc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess ||
      cudaFuncSetAttribute(k_bulk_alloc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return FDMS_ERR_UNSUPPORTED;
  return aw.counts && aw.hdr && aw.amax ? FDMS_OK : FDMS_ERR_CUDA;
}

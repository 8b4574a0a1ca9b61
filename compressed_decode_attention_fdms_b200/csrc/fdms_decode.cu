// Decode attention over the compact store.
//
// FastDMS decodes over the survivors of per-head eviction only, reading 5-8x
// less KV than a dense cache ("FastDMS: 6.4X KV-cache compression running
// faster than vLLM BF16/FP8", aiwitness.kr/community/1t3vlrx, paragraph on
// decode speed and memory at 8K context). For query head g of kv head h:
//     o_g = sum_{j in S_h} softmax_j(scale * q_g . k_j) v_j,
// S_h = the head's compact store plus its visible ring slots.
//
// The kernel is memory bound: every byte of a visible K and V row is read once.
// A tile is 4 KB of K rows and 4 KB of V rows of one 64-slot page (32 rows of
// 128 bytes): a store tile, or a ring frame (TR consecutive positions, which
// sit in TR consecutive ring slots).
//   - Two ways to spread the work, chosen per call on the host:
//     * per-head clusters (calls with few (seq, kv head) pairs): one
//       thread-block cluster of 2-8 CTAs per pair; the head's tiles are dealt
//       over the cluster's warps; the warps' partials (m, l, o) are merged in
//       shared memory, the CTAs' through distributed shared memory, and the
//       cluster writes the output. No plan or workspace.
//     * one plan (other calls): the tiles of all heads of the call are laid
//       end to end and cut into equal ranges, one per warp of the grid, every
//       CTA that can be resident at once (two per SM here). A warp that
//       covers a whole head writes its output; otherwise
//       it leaves a partial, and the last warp of the head to finish (a
//       per-head arrival counter) merges the head's partials.
//   - The store is append-only and a ring slot keeps its row until the ring
//     wraps past it, so everything a decode call saw of a head stays where it
//     was. Each decode leaves a per-head snapshot (length, position, resolved
//     count); the next decode of the same layer plans its tiles from it and
//     issues the copies of those tiles before its dependency wait, while the
//     kernel before it still runs. After the wait it reads the head's current
//     lengths, masks ring rows that have been resolved since, and adds tiles
//     for what is new: in cluster mode by extending the warps' tile lists, in
//     plan mode from spare tile slots the plan set aside for the tokens
//     appended since the snapshot.
//   - Each warp stages its own tiles: K rows, V rows and the head's q go to
//     shared memory by 1-D bulk copies (cp.async.bulk, completion on an
//     mbarrier) into one of the warp's two stages; the warp refills a stage as
//     soon as it has read it. Rows keep their page row in shared memory, so
//     the chunk permutation they are stored with makes the matrix loads free
//     of bank conflicts.
//   - Tile arithmetic on the tensor cores (mma.sync m16n8k16, fp32
//     accumulate), keys on the M side: S^T = K Q^T with 16 keys per MMA row
//     block and the kv head's G query heads as columns; online softmax in fp32
//     in the log2 domain per column; O^T += V^T P^T with 16 head dims per MMA
//     row block. P is carried as a 16-bit head plus a 16-bit remainder, so its
//     rounding stays below 2^-16 relative: with G <= 4 the remainder rides in
//     the MMA's spare columns (column c < G: head of p for head c, G <= c < 2G:
//     remainder of p for head c - G, their sum taken at the end), with G = 8 in
//     a second MMA. The score accumulators are moved into the layout of P^T by
//     an in-register transpose (movmatrix). FP8 pages are converted exactly to
//     f16 (cvt e4m3x2 -> f16x2) and q is brought into f16 range by a power of
//     two that the score scale undoes; the page's K scale multiplies the
//     scores and its V scale the probabilities, never the elements.
//   - Every kernel allows programmatic dependent launch: set-up that reads no
//     data of the previous kernel runs while that kernel finishes.
#include <algorithm>
#include <cfloat>
#include <cstdio>
#include <mutex>

#include "fdms_internal.cuh"

namespace fdms {
namespace {

#ifndef FDMS_CLUSTER_DECODE
#define FDMS_CLUSTER_DECODE 1
#endif

constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

// tile flags: first / last tile of a head in a warp's list, a ring frame, ring
// rows that may be pending (keep bit decides), bf16 rows of a per-block FP8
// cache (the store's partly filled block, staged, or the ring)
enum : int { kFirst = 1, kLast = 2, kRing = 4, kPending = 8, kBf16 = 16 };

struct TileMeta {
  const uint8_t* ksrc;   // K row of frame row 0 (store: the tile's first row in its
                         // block; ring: the frame's first slot); V rows follow the
                         // block's (or the ring's) K rows
  int hidx;              // head of the call (b * Hkv + h)
  int rows;              // row0 | row1 << 8 | flags << 16: frame rows [row0, row1)
  int p0;                // ring tiles: position of frame row 0
  float ks;              // K scale of the page
  float vrel;            // V scale of the page / the head's V scale
  int pad;
};

// where the merged output goes
struct OutArgs {
  void* out;     // bf16 or fp32 [batch][Hq][D]
  float* lse;    // fp32 [batch][Hq] or null
  int f32;
};

template <int D_, bool FP8_, int G_>
struct Dec {
  static constexpr int D = D_, G = G_;
  static constexpr bool FP8 = FP8_;
  static constexpr int ELT = FP8 ? 1 : 2;
  static constexpr int RB = D * ELT;           // bytes per row
  static constexpr int TR = 4096 / RB;         // rows per tile: 4 KB of K, 4 KB of V
  static constexpr int NCW = G * D >= 1024 ? 4 : 8;   // warps per CTA
  static constexpr int NT = NCW * 32;
  static constexpr int SPW = 2;                // stages per warp
  static constexpr int NSTAGE = NCW * SPW;
  static constexpr int NMR = 64;               // tile descriptors held per warp
  static constexpr int KV_BYTES = TR * RB;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;
  static constexpr int MK = TR / 16;           // 16-key row blocks per tile
  static constexpr int KS = D / 16;            // score k-steps (16 dims each)
  static constexpr int MT = D / 16;            // P.V row blocks (16 dims each)
  static constexpr bool PACK = G <= 4;         // p remainder in the spare MMA columns
  static_assert(TR >= 16 && TR <= 64 && 64 % TR == 0, "tiles tile a page");

  static constexpr int OFF_META = NSTAGE * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_META + NCW * NMR * (int)sizeof(TileMeta);
  static constexpr int OFF_HEADS = OFF_BAR + NSTAGE * 8;
  // 32 ints of head state, then one slot of (o [G][D], m [G], l [G]) per warp
  // and one for the CTA
  static constexpr int SLOT = G * D + 2 * G;   // floats
  static constexpr int OFF_MERGE = OFF_HEADS + 128;
  // then the head's block-table row (and FP8 scale pairs), max_blocks entries
  static constexpr int OFF_BT = (OFF_MERGE + (NCW + 1) * SLOT * 4 + 15) / 16 * 16;
  static size_t smem_bytes_cluster(int max_blocks) {
    return 128 + OFF_BT + (size_t)max_blocks * 4 * (FP8 ? 3 : 1) + 64;
  }
  // head dim of P.V accumulator row block i, lane group g, upper half hi:
  // BF16 V^T comes from transposed 8x8 matrix loads (dims in order), FP8 V^T
  // from byte pairs (dims 2g and 2g + 1 of the 16-dim chunk)
  __host__ __device__ static int vdim(int i, int g, int hi) {
    return FP8 ? 16 * i + 2 * g + hi : 16 * i + 8 * hi + g;
  }
};

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for an mbarrier phase, giving up after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > kWaitLimitNs) return false;
  }
}

// Tiles of one head: its store pages (tile = TR rows of a page), then the
// TR-position frames its ring slots r .. n-1 fall in.
template <int TR>
__device__ __forceinline__ int head_tiles(int len, int n, int r) {
  const int live = n - r;
  return (len + TR - 1) / TR + (live > 0 ? (live + (r % TR) + TR - 1) / TR : 0);
}
// Tiles per warp for P tiles over n_ranges warps: ceil(P / n_ranges), at least
// 1; an fp64 estimate of the quotient (inv = 1 / n_ranges) made exact by
// integer correction.
__device__ __forceinline__ int tiles_per_warp(int P, int n_ranges, double inv) {
  long long qq = (long long)((double)P * inv);
  while (qq * n_ranges > P) --qq;
  while ((qq + 1) * n_ranges <= P) ++qq;
  const int S = (int)qq + (qq * n_ranges < P ? 1 : 0);
  return S > 1 ? S : 1;
}

// ------------------------------------------------------------ cluster helpers
// All threads of every CTA of the cluster arrive, then wait: shared-memory
// writes before it are visible to every CTA of the cluster after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The same rendezvous without ordering memory: every thread of the cluster has
// got here (its earlier loads have returned their values).
__device__ __forceinline__ void cluster_sync_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n"
               "barrier.cluster.wait.aligned;" ::: "memory");
}
// shared-memory address of `local`'s counterpart in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_addr(const void* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  return remote;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// ------------------------------------------------------------- MMA helpers
template <bool F16>
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}
// four 8x8 16-bit matrices from shared memory; lane i gives the address of row
// i % 8 of matrix i / 8, register j receives matrix j
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// the same, each matrix transposed
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// transpose of an 8x8 16-bit matrix held one 32-bit pair per lane (lane 4g + t:
// row g, columns 2t and 2t + 1)
__device__ __forceinline__ uint32_t movm_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// two f32 -> packed 16-bit pair (x0 in the low half), round to nearest even
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float x0, float x1) {
  uint32_t r;
  if constexpr (F16)
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(x1), "f"(x0));
  else
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(x1), "f"(x0));
  return r;
}
template <bool F16>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
  if constexpr (F16) {
    float lo, hi;
    asm("{.reg .f16 a, b;\n mov.b32 {a, b}, %2;\n cvt.f32.f16 %0, a;\n cvt.f32.f16 %1, b;}"
        : "=f"(lo), "=f"(hi) : "r"(w));
    return make_float2(lo, hi);
  } else {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
}
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)two));
  return h;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
// the 16-bit part a P^T column carries: 0 = head, 1 = remainder, 2 = none
__device__ __forceinline__ uint32_t pick16(int role, uint32_t head, uint32_t rem) {
  return role == 0 ? head : (role == 1 ? rem : 0u);
}

// Descriptor of one tile from the head's lengths (store length len, tokens n,
// resolved r): store tile `idx` (kind 0) or ring frame `idx` (kind 1, the TR
// positions from idx * TR). Ring frames keep only positions in [r, n).
template <class T>
__device__ __forceinline__ TileMeta tile_meta(const CacheView& c, long long hi, int hidx,
                                              int kind, int idx, int len, int n, int r,
                                              float hs_k, float hs_v,
                                              const int32_t* bt_row = nullptr,
                                              const float* bs_row = nullptr) {
  constexpr int TR = T::TR, RB = T::RB;
  // the head's block-table row and (K, V) scale pairs: given (a copy in shared
  // memory), or in global memory
  if (!bt_row) bt_row = c.block_table + hi * c.max_blocks;
  if (!bs_row) bs_row = c.bt_scale + hi * c.max_blocks * 2;
  TileMeta mt;
  mt.hidx = hidx;
  mt.pad = 0;
  int row0, row1, flags = 0;
  if (kind == 0) {
    const int j = idx * TR / kBlockSlots;
    row0 = 0;
    row1 = min(TR, len - idx * TR);
    const long long blk = bt_row[j];
    if (T::FP8) {
      mt.ks = bs_row[2 * j];
      mt.vrel = bs_row[2 * j + 1] / hs_v;
    } else {
      mt.ks = mt.vrel = 1.0f;
    }
    mt.ksrc = block_k(c, blk) + (long long)((idx * TR) % kBlockSlots) * RB;
    mt.p0 = 0;
  } else {
    const int f0 = idx * TR;
    // clipped to the frame: a frame wholly below r (resolved since a snapshot
    // planned it) or above n comes out empty
    const int lo = min(max(f0, r), f0 + TR), hi_p = max(lo, min(f0 + TR, n));
    row0 = lo - f0;
    row1 = hi_p - f0;
    flags = kRing | (lo < n - c.W ? kPending : 0);
    mt.ks = hs_k;
    mt.vrel = 1.0f;
    mt.ksrc = ring_k(c, hi) + (long long)(f0 % c.R) * RB;
    mt.p0 = f0;
  }
  mt.rows = row0 | row1 << 8 | flags << 16;
  return mt;
}

// Per-block FP8 cache (FDMS_KV_FP8_E4M3_BLOCK): a head's tiles are its sealed
// store blocks (E4M3, TR rows of T per tile, each page with its own K and V
// scale), then the store's partly filled block, staged in bf16 (kind 3), then
// its ring frames, in bf16 (kind 1); the bf16 tiles use the geometry of T16,
// the BF16 configuration of the same D and G (TR16 rows of 2 D bytes).
template <int TR, int TR16>
__host__ __device__ inline int blk_sealed_tiles(int len) {
  return len / kBlockSlots * (kBlockSlots / TR);
}
template <int TR, int TR16>
__host__ __device__ inline int blk_head_tiles(int len, int n, int r) {
  const int staged = len % kBlockSlots, live = n - r;
  return blk_sealed_tiles<TR, TR16>(len) + (staged + TR16 - 1) / TR16 +
         (live > 0 ? (live + (r % TR16) + TR16 - 1) / TR16 : 0);
}
// Descriptor of bf16 tile idx of a per-block FP8 head: staged rows (kind 3:
// rows idx * TR16 .. of the partly filled block) or ring frame idx (kind 1).
template <class T16>
__device__ __forceinline__ TileMeta tile_meta_b16(const CacheView& c, long long hi, int hidx,
                                                  int kind, int idx, int len, int n, int r) {
  constexpr int TR16 = T16::TR, RB16 = T16::RB;
  TileMeta mt;
  mt.hidx = hidx;
  mt.pad = 0;
  mt.ks = mt.vrel = 1.0f;
  int row0, row1, flags = kBf16;
  if (kind == 3) {
    row0 = 0;
    row1 = max(0, min(TR16, len % kBlockSlots - idx * TR16));
    mt.ksrc = stage_k(c, hi) + (long long)idx * TR16 * RB16;
    mt.p0 = 0;
  } else {
    const int f0 = idx * TR16;
    const int lo = min(max(f0, r), f0 + TR16), hi_p = max(lo, min(f0 + TR16, n));
    row0 = lo - f0;
    row1 = hi_p - f0;
    flags |= kRing | (lo < n - c.W ? kPending : 0);
    mt.ksrc = ring_k(c, hi) + (long long)(f0 % c.R) * RB16;
    mt.p0 = f0;
  }
  mt.rows = row0 | row1 << 8 | flags << 16;
  return mt;
}

// The partial of a head's E4M3 tiles (o8, FP8 accumulator layout: dims
// 16 i + 2 g + hf) and that of its bf16 tiles (o16, BF16 layout: dims
// 16 i + 8 hf + g), of the same columns 2t, 2t + 1, merged into o8:
//     o = 2^(m8 - M) s8 o8 + 2^(m16 - M) o16,  l likewise,  M = max(m8, m16),
// s8 the V unit of the E4M3 partial. Each o16 value moves to the lane of the
// FP8 layout that holds its dim (a lane-group shuffle).
template <int MT>
__device__ __forceinline__ void merge_kinds(float (&o8)[MT][4], float& m0, float& m1, float& L0,
                                            float& L1, float s8, const float (&o16)[MT][4],
                                            float n0, float n1, float K0, float K1, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const float M0 = fmaxf(m0, n0), M1 = fmaxf(m1, n1);
  const float a0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - M0) * s8;
  const float a1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - M1) * s8;
  const float b0 = n0 == -INFINITY ? 0.f : fast_exp2(n0 - M0);
  const float b1 = n1 == -INFINITY ? 0.f : fast_exp2(n1 - M1);
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int d = 2 * g + hf, src = 4 * (d & 7) + t;   // dim 16 i + d in the BF16 layout
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float x0 = __shfl_sync(0xffffffffu, o16[i][e], src);
        const float x1 = __shfl_sync(0xffffffffu, o16[i][2 + e], src);
        const float x = (d >> 3) ? x1 : x0;
        o8[i][2 * hf + e] = o8[i][2 * hf + e] * (e ? a1 : a0) + x * (e ? b1 : b0);
      }
    }
  L0 = (m0 == -INFINITY ? 0.f : L0 * fast_exp2(m0 - M0)) + K0 * b0;
  L1 = (m1 == -INFINITY ? 0.f : L1 * fast_exp2(m1 - M1)) + K1 * b1;
  m0 = M0;
  m1 = M1;
}

// ------------------------------------------------------------ a warp's tiles
// One warp's online softmax over the tiles of one head at a time, and the
// arithmetic of a tile staged in shared memory (K rows, V rows, the head's q).
template <class T>
struct WarpTiles {
  static constexpr int D = T::D, G = T::G, RB = T::RB, TR = T::TR, MK = T::MK, KS = T::KS,
                       MT = T::MT;
  static constexpr bool FP8 = T::FP8, PACK = T::PACK;
  static constexpr int NKL = FP8 ? KS / 2 : KS;   // K matrix loads per row block
  static constexpr int NVL = FP8 ? MT / 2 : MT;   // V matrix loads per row block

  int g, t, role0, role1, qh, lrow, lsub, lx;
  float qscale;
  uint32_t qb[KS][2];              // q B-fragments (column g, k-steps)
  float qmul0, qmul1;              // score multipliers of columns 2t, 2t + 1
  int cur_hidx;
  bool q_raw;                      // qb holds raw bf16 words (fetch_q), not yet prepared
  float m0, m1;                    // running max of columns 2t, 2t + 1
  float l0, l1;                    // this lane's part of their sums
  float oacc[MT][4];               // o^T: [dims of row block i] x [columns 2t, 2t + 1]

  __device__ __forceinline__ void init(int lane, float softmax_scale) {
    g = lane >> 2;
    t = lane & 3;
    // P^T columns 2t and 2t + 1 of this lane: head, remainder or nothing
    role0 = PACK ? (2 * t < G ? 0 : (2 * t < 2 * G ? 1 : 2)) : 0;
    role1 = PACK ? (2 * t + 1 < G ? 0 : (2 * t + 1 < 2 * G ? 1 : 2)) : 0;
    qh = PACK ? g % G : g;   // query head of this lane's q column
    // This lane's row address for a matrix load: row 16 m + 8 ((lane >> 3) & 1)
    // + (lane & 7), chunk cb + (lane >> 4), so registers 0..3 receive the
    // matrices (rows 0-7, chunk cb), (rows 8-15, cb), (rows 0-7, cb + 1),
    // (rows 8-15, cb + 1) of row block m. Row blocks start at multiples of 8
    // rows, so the chunk permutation of the row is that of lane & 7.
    lrow = 8 * ((lane >> 3) & 1) + (lane & 7);
    lsub = lane >> 4;
    lx = RB == 64 ? ((lane & 7) >> 1) & 3 : (lane & 7);
    qscale = softmax_scale * kLog2e;
    qmul0 = qmul1 = 0.f;
    cur_hidx = -1;
    q_raw = false;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
#pragma unroll
    for (int i = 0; i < MT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  }
  // a new head: empty running state
  __device__ __forceinline__ void reset() {
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
#pragma unroll
    for (int i = 0; i < MT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  }
  __device__ __forceinline__ uint32_t lm_addr(uint32_t base, int m, int cb) const {
    return base + (uint32_t)((16 * m + lrow) * RB + 16 * ((cb + lsub) ^ lx));
  }

  // q of kv head `hidx` of the call (its G query heads, qg = their first
  // element in global memory): the raw bf16 words of this lane's fragments,
  // loaded now and brought into the MMA operand form by prep_q at first use,
  // so that the load latency overlaps other work
  __device__ __forceinline__ void fetch_q(const uint16_t* __restrict__ qg, int hidx) {
    cur_hidx = hidx;
    q_raw = true;
#pragma unroll
    for (int s2 = 0; s2 < KS; ++s2) {
      if constexpr (FP8) {
        // k-slots 2t, 2t + 1, 2t + 8, 2t + 9 of k-step s are dims
        // 16 s + 4t .. 16 s + 4t + 3 (the order the E4M3 K matrices give)
        const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(qg + qh * D + 16 * s2 + 4 * t));
        qb[s2][0] = w2.x;
        qb[s2][1] = w2.y;
      } else {
        qb[s2][0] = __ldg(reinterpret_cast<const unsigned int*>(qg + qh * D + 16 * s2 + 2 * t));
        qb[s2][1] = __ldg(reinterpret_cast<const unsigned int*>(qg + qh * D + 16 * s2 + 8 + 2 * t));
      }
    }
  }
  __device__ __forceinline__ void prep_q() {
    q_raw = false;
    if constexpr (FP8) {
      // f16 q scaled by 2^a so that max |q| of the head is in [2^14, 2^15)
      // (bf16 -> f16 is then exact); the four lanes of a lane group hold a
      // whole head
      float amax = 0.f;
#pragma unroll
      for (int s2 = 0; s2 < KS; ++s2)
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(__uint_as_float(qb[s2][0] << 16)),
                                       fabsf(__uint_as_float(qb[s2][0] & 0xFFFF0000u))),
                                 fmaxf(fabsf(__uint_as_float(qb[s2][1] << 16)),
                                       fabsf(__uint_as_float(qb[s2][1] & 0xFFFF0000u)))));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      int ex = 0;
      if (amax > 0.f) ex = 141 - (int)((__float_as_uint(amax) >> 23) & 0xFF);
      ex = max(-126, min(126, ex));
      const float up = __uint_as_float((uint32_t)(ex + 127) << 23);
      const float down = __uint_as_float((uint32_t)(127 - ex) << 23);
      const float qm = qscale * down;
#pragma unroll
      for (int s2 = 0; s2 < KS; ++s2) {
        const uint32_t x = qb[s2][0], y = qb[s2][1];
        qb[s2][0] = pack2<true>(__uint_as_float(x << 16) * up, __uint_as_float(x & 0xFFFF0000u) * up);
        qb[s2][1] = pack2<true>(__uint_as_float(y << 16) * up, __uint_as_float(y & 0xFFFF0000u) * up);
      }
      // column c carries query head c % G (c when G = 8); lane 4c holds its multiplier
      qmul0 = __shfl_sync(0xffffffffu, qm, 4 * (2 * t));
      qmul1 = __shfl_sync(0xffffffffu, qm, 4 * (2 * t + 1));
    } else {
      qmul0 = qmul1 = qscale;
    }
  }

  // The tile staged at Ks (K rows, then V rows) of the head whose q fetch_q
  // loaded. Pending ring rows (positions below thresh) count only when their
  // keep byte (keep[p % R]) is set.
  __device__ __forceinline__ void tile(const uint8_t* Ks, const TileMeta& tm, int thresh,
                                       const uint8_t* keep, int R, int lane) {
    const int row0 = tm.rows & 0xFF, row1 = (tm.rows >> 8) & 0xFF, flags = tm.rows >> 16;
    const uint8_t* Vs = Ks + T::KV_BYTES;
    const uint32_t ks_base = smem_addr(Ks), vs_base = smem_addr(Vs);
    if (q_raw) prep_q();
    if (flags & kFirst) {
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
#pragma unroll
      for (int i = 0; i < MT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    }
    if (row1 <= row0) return;   // an empty tile (a spare with nothing new)

    // ---- visible rows of the tile frame: [row0, row1), less the pending ring
    // rows whose keep bit is 0 (one keep byte per row, read only then)
    const bool pend = (flags & kPending) != 0;
    const bool full_tile = row0 == 0 && row1 == TR && !pend;
    unsigned long long vmask = ~0ull;
    if (!full_tile) {
      vmask = (row1 >= 64 ? ~0ull : (1ull << row1) - 1ull) & ~((1ull << row0) - 1ull);
      if (pend) {
#pragma unroll
        for (int h2 = 0; h2 < (TR + 31) / 32; ++h2) {
          const int row = 32 * h2 + lane;
          bool drop = false;
          if (row < TR && row >= row0 && row < row1) {
            const int p = tm.p0 + row;
            drop = p < thresh && keep[p % R] == 0;
          }
          const unsigned bd = __ballot_sync(0xffffffffu, drop);
          vmask &= ~((unsigned long long)bd << (32 * h2));
        }
      }
    }

    // ---- scores S^T[key][column]: keys 16 m + g (elements 0, 1) and
    // 16 m + g + 8 (elements 2, 3) of row block m, columns 2t and 2t + 1
    float sc[MK][4];
    {
      uint32_t ka[MK][NKL][4];
#pragma unroll
      for (int m = 0; m < MK; ++m)
#pragma unroll
        for (int j = 0; j < NKL; ++j) ldsm_x4(ka[m][j], lm_addr(ks_base, m, 2 * j));
      float acc[MK][4];
#pragma unroll
      for (int m = 0; m < MK; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
      if constexpr (FP8) {
        // load j covers k-steps 2j (registers 0, 1) and 2j + 1 (registers 2, 3);
        // a register holds E4M3 dims 4t .. 4t + 3 of its key row: the low pair
        // is k-slots 2t, 2t + 1, the high pair k-slots 2t + 8, 2t + 9
#pragma unroll
        for (int j = 0; j < NKL; ++j)
#pragma unroll
          for (int hc = 0; hc < 2; ++hc)
#pragma unroll
            for (int m = 0; m < MK; ++m) {
              const uint32_t r0 = ka[m][j][2 * hc], r8 = ka[m][j][2 * hc + 1];
              mma16816<true>(acc[m], e4m3x2_to_f16x2(r0 & 0xFFFF), e4m3x2_to_f16x2(r8 & 0xFFFF),
                             e4m3x2_to_f16x2(r0 >> 16), e4m3x2_to_f16x2(r8 >> 16),
                             qb[2 * j + hc][0], qb[2 * j + hc][1]);
            }
      } else {
        // load s is k-step s: chunks 2s (dims 16s .. 16s + 7) and 2s + 1
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2)
#pragma unroll
          for (int m = 0; m < MK; ++m)
            mma16816<false>(acc[m], ka[m][s2][0], ka[m][s2][1], ka[m][s2][2], ka[m][s2][3],
                            qb[s2][0], qb[s2][1]);
      }
      const float mul0 = qmul0 * tm.ks, mul1 = qmul1 * tm.ks;
#pragma unroll
      for (int m = 0; m < MK; ++m) {
        sc[m][0] = acc[m][0] * mul0;
        sc[m][1] = acc[m][1] * mul1;
        sc[m][2] = acc[m][2] * mul0;
        sc[m][3] = acc[m][3] * mul1;
      }
    }
    if (!full_tile) {
#pragma unroll
      for (int m = 0; m < MK; ++m) {
        if (!((vmask >> (16 * m + g)) & 1ull)) sc[m][0] = sc[m][1] = -INFINITY;
        if (!((vmask >> (16 * m + g + 8)) & 1ull)) sc[m][2] = sc[m][3] = -INFINITY;
      }
    }

    // ---- online softmax per column (the 8 lanes with this t share it). With
    // no visible key so far the reference point is 0: every p is then
    // 2^-inf = 0 and so is the rescale of the (empty) accumulators.
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int m = 0; m < MK; ++m) {
      mx0 = fmaxf(mx0, fmaxf(sc[m][0], sc[m][2]));
      mx1 = fmaxf(mx1, fmaxf(sc[m][1], sc[m][3]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float mr0 = mn0 == -INFINITY ? 0.f : mn0, mr1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = fast_exp2(m0 - mr0), al1 = fast_exp2(m1 - mr1);
    float pr[MK][4];
    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
    for (int m = 0; m < MK; ++m) {
      pr[m][0] = fast_exp2(sc[m][0] - mr0);
      pr[m][1] = fast_exp2(sc[m][1] - mr1);
      pr[m][2] = fast_exp2(sc[m][2] - mr0);
      pr[m][3] = fast_exp2(sc[m][3] - mr1);
      ls0 += pr[m][0] + pr[m][2];
      ls1 += pr[m][1] + pr[m][3];
    }
    l0 = l0 * al0 + ls0;
    l1 = l1 * al1 + ls1;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      oacc[i][0] *= al0;
      oacc[i][1] *= al1;
      oacc[i][2] *= al0;
      oacc[i][3] *= al1;
    }

    // ---- P^T B-fragments: 16-bit head and remainder of p * (page V scale /
    // head V scale), moved from the S^T layout (lane 4g + t: key g, columns
    // 2t, 2t + 1) to the B layout (lane 4g + t: keys 2t, 2t + 1 of column g)
    uint32_t bh[MK][2], bl[MK][2];
#pragma unroll
    for (int m = 0; m < MK; ++m) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {   // keys g (hh = 0) and g + 8 (hh = 1)
        const float p0 = pr[m][2 * hh] * tm.vrel, p1 = pr[m][2 * hh + 1] * tm.vrel;
        const uint32_t hw = pack2<FP8>(p0, p1);
        const float2 hf = unpack2<FP8>(hw);
        const uint32_t rw = pack2<FP8>(p0 - hf.x, p1 - hf.y);
        if constexpr (PACK) {
          const uint32_t x = (pick16(role0, hw, rw) & 0xFFFFu) |
                             (pick16(role1, hw, rw) & 0xFFFF0000u);
          bh[m][hh] = movm_t(x);
          bl[m][hh] = 0u;
        } else {
          bh[m][hh] = movm_t(hw);
          bl[m][hh] = movm_t(rw);
        }
      }
    }

    // ---- o^T += V^T P^T, 16 keys (row block m) per k-step
#pragma unroll
    for (int m = 0; m < MK; ++m) {
#pragma unroll
      for (int j = 0; j < NVL; ++j) {
        uint32_t va[4];
        ldsm_x4_t(va, lm_addr(vs_base, m, 2 * j));
        if constexpr (FP8) {
          // load j covers dim chunks 2j (registers 0, 1) and 2j + 1 (2, 3),
          // each one row block of 16 dims; a transposed register holds the
          // byte pairs (dims 2g, 2g + 1) of keys 2t and 2t + 1: row g of the
          // block is dim 2g, row g + 8 dim 2g + 1
#pragma unroll
          for (int hc = 0; hc < 2; ++hc) {
            const int i = 2 * j + hc;
            const uint32_t x = prmt(va[2 * hc], va[2 * hc + 1], 0x6420);
            const uint32_t y = prmt(va[2 * hc], va[2 * hc + 1], 0x7531);
            const uint32_t a0 = e4m3x2_to_f16x2(x & 0xFFFF), a2 = e4m3x2_to_f16x2(x >> 16);
            const uint32_t a1 = e4m3x2_to_f16x2(y & 0xFFFF), a3 = e4m3x2_to_f16x2(y >> 16);
            mma16816<true>(oacc[i], a0, a1, a2, a3, bh[m][0], bh[m][1]);
            if constexpr (!PACK) mma16816<true>(oacc[i], a0, a1, a2, a3, bl[m][0], bl[m][1]);
          }
        } else {
          // load j is row block j: chunks 2j (dims 16j .. 16j + 7, registers
          // 0, 1) and 2j + 1 (dims 16j + 8 .. 16j + 15, registers 2, 3)
          mma16816<false>(oacc[j], va[0], va[2], va[1], va[3], bh[m][0], bh[m][1]);
          if constexpr (!PACK) mma16816<false>(oacc[j], va[0], va[2], va[1], va[3], bl[m][0],
                                               bl[m][1]);
        }
      }
    }
  }

  // End of a head: the sums of columns 2t and 2t + 1 over the warp (L0, L1)
  // and o with each head's p-head and p-remainder columns added (columns h
  // and h + G); lane 4g + t then holds heads 2t (element 0) and 2t + 1 (1).
  __device__ __forceinline__ void finish(float (&o)[MT][4], float& L0, float& L1) const {
    L0 = l0;
    L1 = l1;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      L0 += __shfl_xor_sync(0xffffffffu, L0, off);
      L1 += __shfl_xor_sync(0xffffffffu, L1, off);
    }
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x = oacc[i][e];
        if constexpr (G == 4) x += __shfl_xor_sync(0xffffffffu, x, 2);
        if constexpr (G == 2) x += __shfl_xor_sync(0xffffffffu, x, 1);
        o[i][e] = x;
      }
    if constexpr (G == 1) {
#pragma unroll
      for (int i = 0; i < MT; ++i) {
        o[i][0] += o[i][1];
        o[i][2] += o[i][3];
      }
    }
  }
};

// The stage of a tile into shared memory: K and V rows [row0, row1) of `mt`.
// phase 0: arrival and copies; 1: copies only, no arrival (before the
// dependency wait); 2: the arrival of a tile whose copies phase 1 issued.
template <class T>
__device__ __forceinline__ void stage_tile(const CacheView& c, uint8_t* kdst, uint64_t* bar,
                                           const TileMeta& mt, int phase) {
  constexpr int RB = T::RB;
  uint8_t* vdst = kdst + T::KV_BYTES;
  const int row0 = mt.rows & 0xFF, row1 = (mt.rows >> 8) & 0xFF;
  const uint32_t nb = row1 > row0 ? (uint32_t)(row1 - row0) * RB : 0u;
  const long long voff = (long long)((mt.rows >> 16) & kRing ? c.R : kBlockSlots) * RB;
  if (phase == 0) mbar_arrive_expect_tx(bar, 2u * nb + c.stall_tx);
  if (phase == 1) mbar_expect_tx(bar, 2u * nb + c.stall_tx);
  if (phase == 2) mbar_arrive_expect_tx(bar, 0u);
  if (phase != 2 && nb > 0) {
    bulk_g2s(kdst + row0 * RB, mt.ksrc + (long long)row0 * RB, nb, bar);
    bulk_g2s(vdst + row0 * RB, mt.ksrc + voff + (long long)row0 * RB, nb, bar);
  }
}

// Zero the V halves of every stage (stale V rows are multiplied by p = 0, so
// they must hold numbers; stale K rows only give scores that are masked), then
// set up the stage barriers. Reads no data of the previous kernel.
template <class T>
__device__ __forceinline__ void init_stages(uint8_t* smem, uint64_t* full, int nstage, int nt,
                                            int tid, int warp, int lane) {
  for (int i = tid; i < nstage * (T::KV_BYTES / 16); i += nt) {
    const int st = i / (T::KV_BYTES / 16), off = i % (T::KV_BYTES / 16);
    reinterpret_cast<uint4*>(smem + st * T::STAGE_BYTES + T::KV_BYTES)[off] =
        make_uint4(0u, 0u, 0u, 0u);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // before any bulk copy
  if (lane < T::SPW) mbar_init(&full[warp * T::SPW + lane], 1);
  fence_mbar_init();
}

// ======================================================= per-head clusters
// One cluster of CS CTAs per (seq, kv head) of the call. With use_snap the
// cluster plans from the head's snapshot (one copy for the cluster, shared
// through distributed shared memory) and issues its first copies before the
// dependency wait; the tiles new since then are dealt round-robin after it.
// The warps' partials are merged in shared memory, the CTAs' through
// distributed shared memory, and the cluster writes the output.
template <class T, int CS, bool BLK>
__global__ void __launch_bounds__(T::NT, 1)
k_decode_split(CacheView c, DecodeWork w, OutArgs oa, int layer, int batch,
               const uint16_t* __restrict__ q, int use_snap) {
  // per-block FP8 (BLK): sealed E4M3 tiles with T, the staged block and the
  // ring in bf16 with T16. A snapshot plans its sealed tiles only (a sealed
  // block never changes; the staged block does, in place): the staged and
  // ring tiles, and the blocks sealed since, are dealt after the wait
  using T16 = Dec<T::D, false, T::G>;
  constexpr int TR16 = T16::TR;
  constexpr int D = T::D, G = T::G, TR = T::TR, SPW = T::SPW, MT = T::MT, NMR = T::NMR,
                NCW = T::NCW;
  constexpr bool FP8 = T::FP8;
  constexpr int NW = CS * NCW;              // warps of the cluster
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long hi0 = (long long)layer * c.Bmax * c.Hkv;   // first head of this layer
  TileMeta* ring = reinterpret_cast<TileMeta*>(smem + T::OFF_META) + warp * NMR;
  (void)batch;
  init_stages<T>(smem, full, T::NSTAGE, T::NT, tid, warp, lane);
  auto stg = [&](uint8_t* dst, uint64_t* bar, const TileMeta& mt, int phase) {
    if (BLK && ((mt.rows >> 16) & kBf16)) stage_tile<T16>(c, dst, bar, mt, phase);
    else stage_tile<T>(c, dst, bar, mt, phase);
  };

  const int hsel = (int)(blockIdx.x / CS), crank = (int)(blockIdx.x % CS);
  const int v = crank * NCW + warp;
  const long long hi = hi0 + hsel;
  // cst: [8..10] the lengths the plan is made on (snapshot, or now), [12..14]
  // the lengths now, floats [16..17] FP8 head scales (K, V)
  int* cst = reinterpret_cast<int*>(smem + T::OFF_HEADS);
  float* hs = reinterpret_cast<float*>(cst) + 16;
  float* mslot = reinterpret_cast<float*>(smem + T::OFF_MERGE);
  // the head's block-table row and scale pairs, copied to shared memory in the
  // background from the start; entries of blocks the snapshot already held are
  // final (the store is append-only), later ones are read again after the wait
  int32_t* s_bt = reinterpret_cast<int32_t*>(smem + T::OFF_BT);
  float* s_bs = reinterpret_cast<float*>(s_bt + c.max_blocks);
  {
    const int32_t* gbt = c.block_table + hi * c.max_blocks;
    const float* gbs = c.bt_scale + hi * c.max_blocks * 2;
    for (int j = tid; j < c.max_blocks; j += T::NT) {
      cp_async4(&s_bt[j], gbt + j);
      if (FP8) {
        cp_async4(&s_bs[2 * j], gbs + 2 * j);
        cp_async4(&s_bs[2 * j + 1], gbs + 2 * j + 1);
      }
    }
  }
  int sp_s = 0, f0_s = 0, a_first = 0, cnt = 0, e0 = 0, E_store = 0, fx0 = 0, nt = 0;
  unsigned pre_mask = 0;
  // warp v's snapshot tiles: a run of the head's tiles, runs differing by at
  // most one; the tiles new since the snapshot continue the round
  auto split = [&](int len_s, int n_s, int r_s) {
    sp_s = (len_s + TR - 1) / TR;
    f0_s = r_s / TR;
    const int P_s = !BLK ? head_tiles<TR>(len_s, n_s, r_s)
                         : (use_snap ? blk_sealed_tiles<TR, TR16>(len_s)
                                     : blk_head_tiles<TR, TR16>(len_s, n_s, r_s));
    const int qq = P_s / NW, rem = P_s % NW;
    cnt = qq + (v < rem ? 1 : 0);
    a_first = v * qq + min(v, rem);
    e0 = (v - rem + NW) % NW;
  };
  // snapshot tile k of this warp: store tile or ring frame, and whether it
  // can still grow (the last store tile and the last ring frame when partly
  // filled)
  auto snap_item = [&](int k, int& kind, int& idx) -> bool {
    const int item = a_first + k;
    if (BLK) {   // a sealed tile: final
      kind = 0;
      idx = item;
      return false;
    }
    kind = item < sp_s ? 0 : 1;
    idx = kind == 0 ? item : f0_s + (item - sp_s);
    const int len_s = cst[8], n_s = cst[9];
    return kind == 0 ? (idx == sp_s - 1 && len_s % TR != 0)
                     : (idx == (n_s - 1) / TR && n_s % TR != 0);
  };
  // warm L2 with the head's block-table row and lengths (read after the wait)
  if (warp == NCW - 1) {
    const char* btp = reinterpret_cast<const char*>(c.block_table + hi * c.max_blocks);
    for (int i = lane; i * 128 < c.max_blocks * 4; i += 32)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(btp + i * 128));
    if (lane == 0) {
      asm volatile("prefetch.global.L2 [%0];" ::"l"(c.store_len + hi));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(c.tok_n + hi));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(c.tok_r + hi));
    }
  }
  if (use_snap) {
    // ---- before the wait: the snapshot and the head scales (fixed once the
    // head holds a token). Every CTA of the cluster reads the same copy: this
    // call writes the other one
    if (tid == 0) {
      int4 sv = w.snap_rd[hi];
      const float2 sc = FP8 ? *reinterpret_cast<const float2*>(c.head_scale + hi * 2)
                            : make_float2(1.f, 1.f);
      if (!(sv.x >= 0 && sv.x <= sv.z && sv.z <= sv.y && sv.y <= c.max_seq_len &&
            sv.y - sv.z <= c.R))
        sv = make_int4(0, 0, 0, 0);
      cst[8] = sv.x;
      cst[9] = sv.y;
      cst[10] = sv.z;
      hs[0] = sc.x;
      hs[1] = sc.y;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // this thread's block-table copies
    __syncthreads();
    const int len_s = cst[8], n_s = cst[9], r_s = cst[10];
    // BLK: the V unit of the E4M3 tiles is the first sealed block's V scale
    // (final once sealed)
    const float hs_k = BLK ? 1.0f : hs[0];
    const float hs_v = BLK ? (len_s >= kBlockSlots ? s_bs[1] : 1.0f) : hs[1];
    split(len_s, n_s, r_s);
    // copies of the warp's first tiles, unless they can still grow
    bool pre = false;
    if (lane < SPW && lane < cnt) {
      int kind, idx;
      if (!snap_item(lane, kind, idx)) {
        TileMeta mt =
            tile_meta<T>(c, hi, hsel, kind, idx, len_s, n_s, r_s, hs_k, hs_v, s_bt, s_bs);
        mt.rows |= (lane == 0 ? kFirst : 0) << 16;
        ring[lane] = mt;
        stg(smem + (warp * SPW + lane) * T::STAGE_BYTES, &full[warp * SPW + lane],
                      mt, 1);
        pre = true;
      }
    }
    pre_mask = __ballot_sync(0xffffffffu, pre);
  }
  WarpTiles<T> wt;
  wt.init(lane, c.softmax_scale);
  WarpTiles<T16> wt16;   // the bf16 tiles of a per-block FP8 head
  if (BLK) wt16.init(lane, c.softmax_scale);
  pdl_wait();                 // the previous kernel's writes are visible from here on
  pdl_launch_dependents();
  // q (an input of this call) and the arrivals of the tiles issued early
  const uint16_t* qh = q + ((long long)(hsel / c.Hkv) * c.Hq + (long long)(hsel % c.Hkv) * G) * D;
  wt.fetch_q(qh, hsel);
  if (BLK) wt16.fetch_q(qh, hsel);
  if ((pre_mask >> lane) & 1)
    stg(smem + (warp * SPW + lane) * T::STAGE_BYTES, &full[warp * SPW + lane],
                  ring[lane], 2);
  if (tid == 0) {
    const int len = c.store_len[hi], n = c.tok_n[hi], r = c.tok_r[hi];
    cst[12] = len;
    cst[13] = n;
    cst[14] = r;
    if (BLK) {   // the V unit of the E4M3 tiles: the first sealed block's V scale
      hs[0] = 1.0f;
      hs[1] = len >= kBlockSlots ? c.bt_scale[hi * c.max_blocks * 2 + 1] : 1.0f;
    } else if (!use_snap || cst[9] == 0) {
      hs[0] = FP8 ? c.head_scale[hi * 2] : 1.0f;
      hs[1] = FP8 ? c.head_scale[hi * 2 + 1] : 1.0f;
    }
    if (!use_snap) {
      cst[8] = len;
      cst[9] = n;
      cst[10] = r;
    }
    if (crank == 0) {
      w.snap_wr[hi] = make_int4(len, n, r, 0);
      atomicAdd(&c.ctr->slots_decoded, (unsigned long long)(len + (n - r)));
      atomicAdd(&c.ctr->bytes_decoded, head_kv_bytes(c, len, n, r));
      if (blockIdx.x == 0) atomicAdd(&c.ctr->decode_calls, 1ull);
    }
  }
  __syncthreads();
  {
    // block-table entries the copy may have missed: every one without a
    // snapshot, else those of blocks added since (BLK: sealed since; the
    // staged block has no entry until it is sealed)
    const int nb_ok = !use_snap ? 0
                      : BLK     ? cst[8] / kBlockSlots
                                : (cst[8] + kBlockSlots - 1) / kBlockSlots;
    const int nb_now = (cst[12] + kBlockSlots - 1) / kBlockSlots;
    if (!use_snap) asm volatile("cp.async.wait_all;" ::: "memory");
    if (nb_now > nb_ok) {
      for (int j = nb_ok + tid; j < nb_now; j += T::NT) {
        s_bt[j] = c.block_table[hi * c.max_blocks + j];
        if (FP8) {
          s_bs[2 * j] = c.bt_scale[(hi * c.max_blocks + j) * 2];
          s_bs[2 * j + 1] = c.bt_scale[(hi * c.max_blocks + j) * 2 + 1];
        }
      }
    }
    __syncthreads();
  }
  {
    const int len_s = cst[8], n_s = cst[9], r_s = cst[10];
    const int len = cst[12], n = cst[13], r = cst[14];
    if (!use_snap) split(len_s, n_s, r_s);
    // tiles new since the snapshot: store tiles past its last one, ring frames
    // past its last one (and not below the current first)
    const int sp_c = (len + TR - 1) / TR;
    E_store = max(0, sp_c - sp_s);
    const int nfr_s = head_tiles<TR>(0, n_s, r_s);
    fx0 = max(nfr_s > 0 ? f0_s + nfr_s : r / TR, r / TR);
    const int E_ring = n > r ? max(0, (n - 1) / TR - fx0 + 1) : 0;
    int E = E_store + E_ring;
    if (BLK) {   // without a snapshot the split covers every tile; with one, the
                 // blocks sealed since, the staged tiles and the ring frames are new
      const int live = n - r;
      E = !use_snap ? 0
                    : (blk_sealed_tiles<TR, TR16>(len) - blk_sealed_tiles<TR, TR16>(len_s)) +
                          (len % kBlockSlots + TR16 - 1) / TR16 +
                          (live > 0 ? (live + (r % TR16) + TR16 - 1) / TR16 : 0);
    }
    nt = cnt + (E > e0 ? (E - e0 + NW - 1) / NW : 0);
  }
  if (lane < G) {   // an empty partial until the warp's last tile replaces it
    mslot[warp * T::SLOT + G * D + lane] = -INFINITY;
    mslot[warp * T::SLOT + G * D + G + lane] = 0.f;
  }

  // descriptor of this warp's tile k, from the lengths now
  auto make_meta = [&](int k) -> TileMeta {
    const int len = cst[12], n = cst[13], r = cst[14];
    int kind, idx;
    if (BLK) {   // sealed tiles, staged tiles (kind 3), ring frames of TR16 positions
      const int n8 = blk_sealed_tiles<TR, TR16>(len);
      const int nst = (len % kBlockSlots + TR16 - 1) / TR16;
      // without a snapshot: item a_first + k of the whole list; with one: a
      // sealed tile of the snapshot, or new tile e of [sealed since, staged, ring]
      const int n8s = use_snap ? blk_sealed_tiles<TR, TR16>(cst[8]) : 0;
      int item = a_first + k;
      if (use_snap && k >= cnt) item = n8s + e0 + (k - cnt) * NW;
      if (item < n8) { kind = 0; idx = item; }
      else if (item < n8 + nst) { kind = 3; idx = item - n8; }
      else { kind = 1; idx = r / TR16 + (item - n8 - nst); }
    } else if (k < cnt) {
      const int item = a_first + k;
      kind = item < sp_s ? 0 : 1;
      idx = kind == 0 ? item : f0_s + (item - sp_s);
    } else {
      const int e = e0 + (k - cnt) * NW;
      kind = e < E_store ? 0 : 1;
      idx = kind == 0 ? sp_s + e : fx0 + (e - E_store);
    }
    TileMeta mt = (BLK && kind != 0)
                      ? tile_meta_b16<T16>(c, hi, hsel, kind, idx, len, n, r)
                      : tile_meta<T>(c, hi, hsel, kind, idx, len, n, r, hs[0], hs[1], s_bt, s_bs);
    mt.rows |= ((k == 0 ? kFirst : 0) | (k == nt - 1 ? kLast : 0)) << 16;
    return mt;
  };
  auto fill = [&](int k0) {   // descriptors of tiles [k0, k0 + 32) into the warp's ring
    const int k = k0 + lane;
    if (k < nt) ring[k % NMR] = make_meta(k);
  };
  fill(0);
  fill(32);
  __syncwarp();
  if (lane < SPW && lane < nt && !((pre_mask >> lane) & 1))
    stg(smem + (warp * SPW + lane) * T::STAGE_BYTES, &full[warp * SPW + lane],
                  ring[lane], 0);

  // ================= tiles of this warp
  const uint8_t* keep = c.ring_keep + hi * c.Rpad;
  const int thresh = cst[13] - c.W;
  for (int k = 0; k < nt; ++k) {
    const int s = warp * SPW + (k % SPW);
    const bool ok = mbar_wait(&full[s], (k / SPW) & 1);
    if (!__all_sync(0xffffffffu, ok)) {
      // a copy did not land in time: latch the error, give the warp's other
      // stage in flight one more bounded wait so that no copy is left pending
      // into shared memory when the CTA leaves, and stop
      if (lane == 0) {
        latch_error(c.ctr, FDMS_ERR_DEVICE);
        if (k + 1 < nt) mbar_wait(&full[warp * SPW + ((k + 1) % SPW)], ((k + 1) / SPW) & 1);
      }
      __syncwarp();
      break;
    }
    const TileMeta tm = ring[k % NMR];
    if (BLK && ((tm.rows >> 16) & kBf16))
      wt16.tile(smem + s * T::STAGE_BYTES, tm, thresh, keep, c.R, lane);
    else
      wt.tile(smem + s * T::STAGE_BYTES, tm, thresh, keep, c.R, lane);
    __syncwarp();
    // descriptors come 32 at a time: those of tiles k + 33 .. k + 64 once
    // tile k + 1 starts a new 32
    if ((k + 1) % 32 == 0 && k + 33 < nt) {
      fill(k + 33);
      __syncwarp();
    }
    // the stage is free: refill it with tile k + SPW
    if (lane == 0 && k + SPW < nt)
      stg(smem + s * T::STAGE_BYTES, &full[s], ring[(k + SPW) % NMR], 0);
    if ((tm.rows >> 16) & kLast) {   // the warp's partial, for the CTA's merge
      float o[MT][4], L0, L1;
      wt.finish(o, L0, L1);
      float vhead = hs[1];
      if constexpr (BLK) {   // the bf16 tiles' partial joins, in the E4M3 layout and V unit 1
        float o16[MT][4], K0, K1;
        wt16.finish(o16, K0, K1);
        merge_kinds<MT>(o, wt.m0, wt.m1, L0, L1, vhead, o16, wt16.m0, wt16.m1, K0, K1, lane);
        vhead = 1.0f;
      }
      float* po = mslot + warp * T::SLOT;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = 2 * wt.t + e;
        if (h >= G) continue;
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          po[h * D + T::vdim(i, wt.g, 0)] = o[i][e] * vhead;
          po[h * D + T::vdim(i, wt.g, 1)] = o[i][2 + e] * vhead;
        }
        if (wt.g == 0) {
          po[G * D + h] = e ? wt.m1 : wt.m0;
          po[G * D + G + h] = e ? L1 : L0;
        }
      }
    }
  }

  // ---- merge: the warps' partials into the CTA's (shared memory), then the
  // CTAs' partials across the cluster; each CTA writes 1/CS of the head's
  // output. o = sum_w 2^(m_w - M) o_w / sum_w 2^(m_w - M) l_w.
  __syncthreads();
  float* cpart = mslot + NCW * T::SLOT;
  for (int e = tid; e < G * D; e += T::NT) {
    const int h = e / D;
    float mv[NCW], M = -INFINITY;
#pragma unroll
    for (int u = 0; u < NCW; ++u) {
      mv[u] = mslot[u * T::SLOT + G * D + h];
      M = fmaxf(M, mv[u]);
    }
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int u = 0; u < NCW; ++u) {
        if (mv[u] != -INFINITY) {   // empty partials hold no o values
          const float bw = fast_exp2(mv[u] - M);
          L += mslot[u * T::SLOT + G * D + G + h] * bw;
          O += mslot[u * T::SLOT + e] * bw;
        }
      }
    }
    cpart[e] = O;
    if (e % D == 0) {
      cpart[G * D + h] = M;
      cpart[G * D + G + h] = L;
    }
  }
  __syncthreads();   // converged warps for the aligned cluster barrier
  cluster_sync_all();
  uint32_t rbase[CS];
#pragma unroll
  for (int j = 0; j < CS; ++j) rbase[j] = cluster_addr(cpart, (uint32_t)j);
  const int kb = hsel / c.Hkv, kh = hsel % c.Hkv;
  constexpr int PER = G * D / CS;
  for (int e = crank * PER + tid; e < (crank + 1) * PER; e += T::NT) {
    const int h = e / D, d = e % D;
    float mj[CS], lj[CS], oj[CS];
#pragma unroll
    for (int j = 0; j < CS; ++j) {   // every load first, then the arithmetic
      mj[j] = ld_dsmem_f32(rbase[j] + 4u * (uint32_t)(G * D + h));
      lj[j] = ld_dsmem_f32(rbase[j] + 4u * (uint32_t)(G * D + G + h));
      oj[j] = ld_dsmem_f32(rbase[j] + 4u * (uint32_t)e);
    }
    float M = -INFINITY;
#pragma unroll
    for (int j = 0; j < CS; ++j) M = fmaxf(M, mj[j]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int j = 0; j < CS; ++j) {
        const float bw = mj[j] == -INFINITY ? 0.f : fast_exp2(mj[j] - M);
        L += lj[j] * bw;
        O += oj[j] * bw;
      }
    }
    const float o = M == -INFINITY ? 0.f : O / L;
    const long long oi = ((long long)kb * c.Hq + (long long)kh * G + h) * D + d;
    if (oa.f32) static_cast<float*>(oa.out)[oi] = o;
    else static_cast<uint16_t*>(oa.out)[oi] = f32_to_bf16_rn(o);
    if (oa.lse && d == 0)
      oa.lse[(long long)kb * c.Hq + kh * G + h] =
          M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
  }
  __syncwarp();
  cluster_sync_relaxed();   // no CTA leaves while another still reads its shared memory
}

// float vectors of 2 or 4 lanes for the partial merge
template <int VW> struct FVec;
template <> struct FVec<2> {
  float x[2];
  __device__ __forceinline__ void load(const float* p) {
    const float2 v = __ldcg(reinterpret_cast<const float2*>(p));
    x[0] = v.x;
    x[1] = v.y;
  }
};
template <> struct FVec<4> {
  float x[4];
  __device__ __forceinline__ void load(const float* p) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(p));
    x[0] = v.x;
    x[1] = v.y;
    x[2] = v.z;
    x[3] = v.w;
  }
};

// One warp merges the np partials (m, l, o) of head h that sit at parts
// p0 .. p0 + np - 1 of the workspace and writes the head's output:
//     o = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p,  M = max_p m_p
// (per query head). Lane i owns elements [i E, i E + E) of the head's G x D
// output, all of one query head. The loads of a batch of parts are issued
// together and unconditionally (a part past the end is read again with weight
// 0): the merge costs one L2 round trip per batch, the (m, l) pairs included.
template <class T>
__device__ __forceinline__ void merge_parts(const CacheView& c, const DecodeWork& w,
                                            const OutArgs& oa, int h, long long p0, int np,
                                            int lane) {
  constexpr int G = T::G, D = T::D, E = G * D / 32, VW = E >= 4 ? 4 : E, NV = E / VW;
  constexpr int PB = E <= 4 ? 24 : (E <= 8 ? 12 : 64 / E);   // parts per batch of loads
  const int hq_l = lane * E / D, d0 = (lane * E) % D;
  float Mc[G], Lc[G], acc[E];
#pragma unroll
  for (int q = 0; q < G; ++q) {
    Mc[q] = -INFINITY;
    Lc[q] = 0.f;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int c0 = 0; c0 < np; c0 += 32) {
    const int cn = min(32, np - c0);
    // (m, l) of part c0 + lane, one pair per query head, and the first batch
    // of partial sums, in one round trip
    float2 ml[G];
    {
      const float2* src = reinterpret_cast<const float2*>(w.part_ml) +
                          (p0 + c0 + min(lane, cn - 1)) * G;
#pragma unroll
      for (int q = 0; q < G; ++q) ml[q] = __ldcg(src + q);
    }
    FVec<VW> ov[PB][NV];
    auto load_batch = [&](int pb) {
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const float* src =
            w.part_o + (p0 + c0 + min(pb + u, cn - 1)) * (long long)(G * D) + lane * E;
#pragma unroll
        for (int j = 0; j < NV; ++j) ov[u][j].load(src + j * VW);
      }
    };
    load_batch(0);
    float wq[G];
    float al = 1.f;
#pragma unroll
    for (int q = 0; q < G; ++q) {
      const float m = lane < cn ? ml[q].x : -INFINITY, l = lane < cn ? ml[q].y : 0.f;
      float mx = m;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float Mn = fmaxf(Mc[q], mx), ref = Mn == -INFINITY ? 0.f : Mn;
      const float a = fast_exp2(Mc[q] - ref);   // 0 while nothing was merged
      wq[q] = fast_exp2(m - ref);               // 0 for an empty partial
      float ls = wq[q] * l;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
      Lc[q] = Lc[q] * a + ls;
      Mc[q] = Mn;
      al = q == hq_l ? a : al;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= al;
    for (int pb = 0; pb < cn; pb += PB) {
      if (pb > 0) load_batch(pb);
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        float ws = 0.f;
#pragma unroll
        for (int q = 0; q < G; ++q) {
          const float x = __shfl_sync(0xffffffffu, wq[q], (pb + u) & 31);
          ws = q == hq_l ? x : ws;
        }
        ws = pb + u < cn ? ws : 0.f;
#pragma unroll
        for (int j = 0; j < NV; ++j)
#pragma unroll
          for (int x = 0; x < VW; ++x) acc[j * VW + x] += ws * ov[u][j].x[x];
      }
    }
  }
  float M = -INFINITY, L = 0.f;
#pragma unroll
  for (int q = 0; q < G; ++q) {
    M = q == hq_l ? Mc[q] : M;
    L = q == hq_l ? Lc[q] : L;
  }
  const float inv = M == -INFINITY ? 0.f : 1.f / L;
  const int kb = h / c.Hkv, kh = h % c.Hkv;
  const long long ob = ((long long)kb * c.Hq + (long long)kh * G + hq_l) * D + d0;
  if (oa.f32) {
    float* dst = static_cast<float*>(oa.out) + ob;
#pragma unroll
    for (int j = 0; j < E; j += VW) {
      if constexpr (VW == 4)
        *reinterpret_cast<float4*>(dst + j) =
            make_float4(acc[j] * inv, acc[j + 1] * inv, acc[j + 2] * inv, acc[j + 3] * inv);
      else
        *reinterpret_cast<float2*>(dst + j) = make_float2(acc[j] * inv, acc[j + 1] * inv);
    }
  } else {
    // E bf16 values, packed two per word, stored 8, 4 or 2 at a time
    uint32_t pk[E / 2];
#pragma unroll
    for (int j = 0; j < E / 2; ++j)
      pk[j] = (uint32_t)f32_to_bf16_rn(acc[2 * j] * inv) |
              ((uint32_t)f32_to_bf16_rn(acc[2 * j + 1] * inv) << 16);
    uint16_t* dst = static_cast<uint16_t*>(oa.out) + ob;
#pragma unroll
    for (int j = 0; j < E / 2; j += (E >= 8 ? 4 : E / 2)) {
      if constexpr (E >= 8)
        *reinterpret_cast<uint4*>(dst + 2 * j) = make_uint4(pk[j], pk[j + 1], pk[j + 2], pk[j + 3]);
      else if constexpr (E == 4)
        *reinterpret_cast<uint2*>(dst + 2 * j) = make_uint2(pk[j], pk[j + 1]);
      else
        *reinterpret_cast<uint32_t*>(dst + 2 * j) = pk[j];
    }
  }
  if (oa.lse && d0 == 0)
    oa.lse[(long long)kb * c.Hq + kh * G + hq_l] =
        M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
}

// ============================================================ global plan
// Every head of the call laid end to end, then cut into equal tile ranges, one
// per warp of the grid. A CTA holds PW warps and is small enough (about 110
// KB of shared memory) for two to share an SM, so that a call's copies go out
// while the call before it still computes.
//   - With use_snap the plan is made from every head's snapshot before the
//     dependency wait: each head gets its snapshot tiles plus `spare` tiles
//     for what it can have gained since (tok_since tokens per sequence
//     appended since that decode and the resolution period bound it); the
//     store tiles below the snapshot's last partial one keep their
//     descriptors and the warps' first copies go out before the wait. After
//     the wait the spares become the new tiles or stay empty.
//   - A head that lies within one warp's range is written by that warp.
//     Otherwise each warp that covered part of it writes a partial (m, l, o)
//     and counts it on the head's counter; the warp that brings the count to
//     the number of parts merges them,
//         o = sum_w 2^(m_w - M) o_w / sum_w 2^(m_w - M) l_w,
//     writes the output and resets the counter.
//   - The last CTA to finish writes the snapshot of every head of the call.
template <class T, int NW>
struct PlanL {
  static constexpr int NT = NW * 32, SPW = T::SPW, NSTAGE = NW * SPW, NMR = 32, HALF = NMR / 2;
  static constexpr int OFF_META = NSTAGE * T::STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_META + NW * NMR * (int)sizeof(TileMeta);   // + lengths barrier
  static constexpr int OFF_MISC = OFF_BAR + NSTAGE * 8 + 8;
  static constexpr int OFF_HEADS = (OFF_MISC + 64 + 15) / 16 * 16;
  // per head: tile prefix (nh + 1), lengths now len, n, r, snapshot len, n, r,
  // FP8 scales (K, V)
  static size_t smem_bytes(int nh) {
    return 128 + OFF_HEADS + (size_t)(nh + 1) * 4 + (size_t)nh * 32 + 16;
  }
};

// Warps per CTA of the global plan: two CTAs must fit on an SM, in shared
// memory and in registers, whose need per warp grows with G x D (the merge's
// loads and the accumulators).
template <class T>
struct PlanWarps {
  static constexpr int value = T::G * T::D >= 1024 ? 4 : (T::G * T::D > 256 ? 5 : 6);
};

template <class T, int NW, bool BLK>
__global__ void __launch_bounds__(NW * 32, 2)
k_decode_plan(CacheView c, DecodeWork w, OutArgs oa, int layer, int batch,
              const uint16_t* __restrict__ q, int n_ranges, double inv_ranges, int use_snap,
              int tok_since) {
  using PL = PlanL<T, NW>;
  // per-block FP8 (BLK): sealed E4M3 tiles with T, bf16 tiles with T16; no
  // snapshots (use_snap is 0)
  using T16 = Dec<T::D, false, T::G>;
  constexpr int TR16 = T16::TR;
  constexpr int D = T::D, G = T::G, TR = T::TR, SPW = T::SPW, MT = T::MT, NMR = PL::NMR,
                HALF = PL::HALF, NT = PL::NT;
  constexpr bool FP8 = T::FP8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + PL::OFF_BAR);
  const int NH = batch * c.Hkv;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long hi0 = (long long)layer * c.Bmax * c.Hkv;   // first head of this layer
  TileMeta* ring = reinterpret_cast<TileMeta*>(smem + PL::OFF_META) + warp * NMR;
  int* misc = reinterpret_cast<int*>(smem + PL::OFF_MISC);
  int* page_off = reinterpret_cast<int*>(smem + PL::OFF_HEADS);   // [NH + 1]
  int* cl = page_off + NH + 1;   // lengths now
  int* cn = cl + NH;
  int* cr = cn + NH;
  int* sl = cr + NH;             // lengths the plan is made on: the snapshot's, or
  int* sn = sl + NH;             // without one those now
  int* sr = sn + NH;
  float* hsc = reinterpret_cast<float*>(sr + NH);   // [NH][2]
  if (!use_snap) {
    sl = cl;
    sn = cn;
    sr = cr;
  }
  uint64_t* len_bar = full + PL::NSTAGE;   // the lengths now have landed (every thread arrives)
  if (tid == 0) mbar_init(len_bar, NT);
  init_stages<T>(smem, full, PL::NSTAGE, NT, tid, warp, lane);
  // the copies of a tile (bf16 tiles of a per-block FP8 cache have 2 D-byte rows)
  auto stg = [&](uint8_t* dst, uint64_t* bar, const TileMeta& mt, int phase) {
    if (BLK && ((mt.rows >> 16) & kBf16)) stage_tile<T16>(c, dst, bar, mt, phase);
    else stage_tile<T>(c, dst, bar, mt, phase);
  };

  // warm L2 with this layer's lengths and block tables (read after the wait)
  {
    const long long bt_lines = ((long long)NH * c.max_blocks * 4 + 127) / 128;
    const char* btp = reinterpret_cast<const char*>(c.block_table + hi0 * c.max_blocks);
    for (long long i = (long long)blockIdx.x * NT + tid; i < bt_lines;
         i += (long long)gridDim.x * NT)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(btp + i * 128));
    if (tid < 4 && blockIdx.x < 8) {
      const char* arr = tid == 0   ? reinterpret_cast<const char*>(c.store_len + hi0)
                        : tid == 1 ? reinterpret_cast<const char*>(c.tok_n + hi0)
                        : tid == 2 ? reinterpret_cast<const char*>(c.tok_r + hi0)
                                   : reinterpret_cast<const char*>(c.head_scale + hi0 * 2);
      const int bytes = tid == 3 ? NH * 8 : NH * 4;   // this layer's slice only
      for (int j = blockIdx.x; j * 128 < bytes; j += 8)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(arr + j * 128));
    }
  }

  // spare tiles of a head: new store tiles (the resolved positions grow by at
  // most tok_since + P - 1) and new ring frames (at most tok_since positions,
  // one more frame when the snapshot's ring was empty)
  const int sp_base =
      use_snap ? (tok_since + c.P - 1 + TR - 1) / TR + (tok_since + TR - 1) / TR : 0;
  auto spares = [&](int h) -> int {
    return use_snap ? sp_base + (sn[h] == sr[h] ? 1 : 0) : 0;
  };
  auto htiles = [&](int len, int n, int r) -> int {
    if constexpr (BLK) return blk_head_tiles<TR, TR16>(len, n, r);
    else return head_tiles<TR>(len, n, r);
  };
  auto plan_tiles = [&](int h) -> int { return max(1, htiles(sl[h], sn[h], sr[h]) + spares(h)); };
  // exclusive prefix of the heads' plan tiles (sl, sn, sr filled)
  auto scan = [&]() {
    const int per = (NH + NT - 1) / NT;
    const int h0 = min(NH, tid * per), h1 = min(NH, h0 + per);
    int sp = 0;
    for (int h = h0; h < h1; ++h) sp += plan_tiles(h);
    int ip = sp;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, ip, off);
      if (lane >= off) ip += a;
    }
    if (lane == 31) misc[4 + warp] = ip;
    __syncthreads();
    int ep = ip - sp;
    for (int i = 0; i < warp; ++i) ep += misc[4 + i];
    for (int h = h0; h < h1; ++h) {
      page_off[h] = ep;
      ep += plan_tiles(h);
    }
    if (tid == NT - 1) page_off[NH] = ep;
    __syncthreads();
  };

  int S = 1, gp0 = 0, nt = 0, h_gs = 0, h_ge = 0;
  long long v_range = 0;
  // this warp's tiles [gp0, gp0 + nt) and the heads h_gs .. h_ge they belong
  // to; range v goes to warp v / gridDim.x of CTA v % gridDim.x, so that when
  // fewer ranges than warps hold tiles, the busy ones spread over every SM
  auto ranges = [&]() {
    const int P = page_off[NH];
    S = tiles_per_warp(P, n_ranges, inv_ranges);
    v_range = (long long)warp * gridDim.x + blockIdx.x;
    gp0 = (int)min(v_range * S, (long long)P);
    nt = min(gp0 + S, P) - gp0;
    h_gs = h_ge = 0;
    if (nt > 0) {
      for (int base = 1; base < NH; base += 32) {
        const int h = base + lane;
        const int po = h < NH ? page_off[h] : P;
        h_gs += __popc(__ballot_sync(0xffffffffu, po <= gp0));
        h_ge += __popc(__ballot_sync(0xffffffffu, po <= gp0 + nt - 1));
      }
    }
  };
  // the head of this warp's tile k and the tile's place in it
  auto head_of = [&](int k, int& h, int& lp) {
    const int gp = gp0 + k;
    int lo = h_gs, hi2 = h_ge;   // the last h in [h_gs, h_ge] with page_off[h] <= gp
    while (lo < hi2) {
      const int mid = (lo + hi2 + 1) >> 1;
      if (page_off[mid] <= gp) lo = mid; else hi2 = mid - 1;
    }
    h = lo;
    lp = gp - page_off[h];
  };
  // kind (0 store tile, 1 ring frame, 2 spare) and index of tile lp of head h
  // in the plan; whether it can still grow since the plan's lengths
  auto plan_item = [&](int h, int lp, int& kind, int& idx) -> bool {
    if constexpr (BLK) {   // sealed tiles, staged tiles (kind 3), ring frames
      const int n8 = blk_sealed_tiles<TR, TR16>(sl[h]);
      const int nst = (sl[h] % kBlockSlots + TR16 - 1) / TR16;
      const int nfr = sn[h] > sr[h] ? (sn[h] - sr[h] + sr[h] % TR16 + TR16 - 1) / TR16 : 0;
      if (lp < n8) { kind = 0; idx = lp; }
      else if (lp < n8 + nst) { kind = 3; idx = lp - n8; }
      else if (lp < n8 + nst + nfr) { kind = 1; idx = sr[h] / TR16 + (lp - n8 - nst); }
      else { kind = 2; idx = 0; }
      return true;
    }
    const int sp = (sl[h] + TR - 1) / TR, nfr = head_tiles<TR>(0, sn[h], sr[h]);
    if (lp < sp) {
      kind = 0;
      idx = lp;
      return lp == sp - 1 && sl[h] % TR != 0;
    }
    if (lp < sp + nfr) {
      kind = 1;
      idx = sr[h] / TR + (lp - sp);
      return idx == (sn[h] - 1) / TR && sn[h] % TR != 0;
    }
    kind = 2;
    idx = lp - sp - nfr;
    return true;
  };
  auto flags_of = [&](int k, int h, int lp) -> int {
    return ((k == 0 || lp == 0) ? kFirst : 0) |
           ((k == nt - 1 || gp0 + k + 1 == page_off[h + 1]) ? kLast : 0);
  };

  // tiles k < 32 issued before the wait / described for good before it /
  // described before it (rows still to set)
  unsigned pre_mask = 0, kept_mask = 0, desc_mask = 0;
  if (use_snap) {
    // ---- before the wait: plan on the snapshots
    for (int h = tid; h < NH; h += NT) {
      int4 sv = w.snap_rd[hi0 + h];
      if (!(sv.x >= 0 && sv.x <= sv.z && sv.z <= sv.y && sv.y <= c.max_seq_len &&
            sv.y - sv.z <= c.R))
        sv = make_int4(0, 0, 0, 0);
      sl[h] = sv.x;
      sn[h] = sv.y;
      sr[h] = sv.z;
      // the head scales are fixed once the head holds a token
      const float2 sc = FP8 ? *reinterpret_cast<const float2*>(c.head_scale + (hi0 + h) * 2)
                            : make_float2(1.f, 1.f);
      hsc[2 * h] = sc.x;
      hsc[2 * h + 1] = sc.y;
    }
    __syncthreads();
    scan();
    ranges();
    // descriptors of the snapshot's tiles: those of store tiles below its
    // last partial one hold after the wait (kept), the others get their rows
    // from the lengths then; the first SPW tiles' copies go out now unless
    // they can still grow
    const int k = lane;
    bool kept = false, described = false;
    if (k < nt && k < NMR) {
      int h, lp, kind, idx;
      head_of(k, h, lp);
      const bool grows = plan_item(h, lp, kind, idx);
      if (kind != 2) {
        TileMeta mt = tile_meta<T>(c, hi0 + h, h, kind, idx, sl[h], sn[h], sr[h], hsc[2 * h],
                                   hsc[2 * h + 1]);
        mt.rows |= (k == 0 || lp == 0 ? kFirst : 0) << 16;
        ring[k] = mt;
        described = true;
        kept = kind == 0 && !grows;
        if (k < SPW && !grows) {
          stg(smem + (warp * SPW + k) * T::STAGE_BYTES, &full[warp * SPW + k], mt,
                        1);
          pre_mask |= 1u << k;
        }
      }
    }
    pre_mask = __ballot_sync(0xffffffffu, (pre_mask >> lane) & 1);
    kept_mask = __ballot_sync(0xffffffffu, kept);
    desc_mask = __ballot_sync(0xffffffffu, described);
  }
  __syncthreads();            // the lengths barrier is set up for every thread
  WarpTiles<T> wt;
  wt.init(lane, c.softmax_scale);
  WarpTiles<T16> wt16;   // the bf16 tiles of a per-block FP8 head
  if (BLK) wt16.init(lane, c.softmax_scale);
  // q of the kv head hidx of the call (its first query head's first element)
  auto q_of = [&](int hidx) -> const uint16_t* {
    return q + ((long long)(hidx / c.Hkv) * c.Hq + (long long)(hidx % c.Hkv) * G) * D;
  };
  pdl_wait();                 // the previous kernel's writes are visible from here on
  pdl_launch_dependents();
  // q of the warp's first head (an input of this call), and the arrivals of
  // the tiles issued early
  if (use_snap && nt > 0) {
    int h, lp;
    head_of(0, h, lp);
    wt.fetch_q(q_of(h), h);
  }
  if ((pre_mask >> lane) & 1)
    stg(smem + (warp * SPW + lane) * T::STAGE_BYTES, &full[warp * SPW + lane],
                  ring[lane], 2);
  // ---- lengths now of every head, and the FP8 head scales the snapshot could
  // not give (heads that held no token then): copied to shared memory in the
  // background. A warp waits for them only when it first needs them: for a
  // tile other than a store tile described before the wait, or at the end.
  for (int h = tid; h < NH; h += NT) {
    const long long hh = hi0 + h;
    cp_async4(&cl[h], c.store_len + hh);
    cp_async4(&cn[h], c.tok_n + hh);
    cp_async4(&cr[h], c.tok_r + hh);
    if (!FP8) {
      if (!use_snap) hsc[2 * h] = hsc[2 * h + 1] = 1.0f;
    } else if (BLK) {   // the V unit of the E4M3 tiles: the head's first block's V scale
      hsc[2 * h] = 1.0f;
      cp_async4(&hsc[2 * h + 1], c.bt_scale + hh * c.max_blocks * 2 + 1);
    } else if (!use_snap || sn[h] == 0) {
      cp_async4(&hsc[2 * h], c.head_scale + hh * 2);
      cp_async4(&hsc[2 * h + 1], c.head_scale + hh * 2 + 1);
    }
  }
  cp_async_arrive(len_bar);
  bool have_len = false, len_ok = true;
  auto wait_len = [&]() {   // warp-uniform
    if (have_len) return;
    len_ok = __all_sync(0xffffffffu, mbar_wait(len_bar, 0));
    if (!len_ok && lane == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
    have_len = true;
  };
  if (!use_snap) {
    wait_len();
    // a plan from lengths that did not land would address anything: the CTA
    // then takes no tiles (the error is latched)
    len_ok = __syncthreads_and(len_ok);
    if (len_ok) {
      scan();
      ranges();
    } else {
      nt = 0;
    }
  }

  // descriptor of this warp's tile k, from the lengths now (an empty tile if
  // they did not land); `pre`: ring[k] holds the tile's descriptor made before
  // the wait, whose block it keeps (a store tile only gains rows)
  auto make_meta = [&](int k, bool pre) -> TileMeta {
    int h, lp, kind, idx;
    head_of(k, h, lp);
    plan_item(h, lp, kind, idx);
    const int len = cl[h], n = cn[h], r = cr[h];
    TileMeta mt;
    if (!len_ok) kind = 2;
    if (!BLK && kind == 2 && len_ok) {   // a spare: the first new store tiles, then the new ring frames
      const int sp = (sl[h] + TR - 1) / TR, nfr = head_tiles<TR>(0, sn[h], sr[h]);
      const int E_store = max(0, (len + TR - 1) / TR - sp);
      const int fx = max(nfr > 0 ? sr[h] / TR + nfr : r / TR, r / TR);
      const int E_ring = n > r ? max(0, (n - 1) / TR - fx + 1) : 0;
      if (idx == spares(h) - 1 && E_store + E_ring > spares(h))
        latch_error(c.ctr, FDMS_ERR_DEVICE);   // more new tiles than spares (cannot happen)
      if (idx < E_store) {
        kind = 0;
        idx = sp + idx;
      } else if (idx < E_store + E_ring) {
        kind = 1;
        idx = fx + (idx - E_store);
      }
    }
    if (kind == 2) {   // an empty tile
      mt.ksrc = nullptr;
      mt.hidx = h;
      mt.rows = 0;
      mt.p0 = 0;
      mt.ks = mt.vrel = 1.0f;
      mt.pad = 0;
    } else if (kind == 0 && pre) {
      mt = ring[k];
      mt.rows = min(TR, len - idx * TR) << 8;
    } else if (BLK && kind != 0) {
      mt = tile_meta_b16<T16>(c, hi0 + h, h, kind, idx, len, n, r);
    } else {
      mt = tile_meta<T>(c, hi0 + h, h, kind, idx, len, n, r, hsc[2 * h], hsc[2 * h + 1]);
    }
    mt.rows = (mt.rows & ~((kFirst | kLast) << 16)) | (flags_of(k, h, lp) << 16);
    return mt;
  };
  // descriptors of tiles [k0, k0 + cnt) into the warp's ring (cnt <= 32)
  auto fill = [&](int k0, int count) {
    const int k = k0 + lane;
    if (lane < count && k < nt) ring[k % NMR] = make_meta(k, false);
  };
  // tiles 0 .. 31 whose descriptors are still to be made from the lengths now;
  // those described before the wait only get their flags
  unsigned todo = (nt >= 32 ? 0xffffffffu : ((1u << nt) - 1u)) & ~kept_mask;
  if ((kept_mask >> lane) & 1) {
    int h, lp;
    head_of(lane, h, lp);
    TileMeta mt = ring[lane];
    mt.rows = (mt.rows & ~((kFirst | kLast) << 16)) | (flags_of(lane, h, lp) << 16);
    ring[lane] = mt;
  }
  __syncwarp();
  auto ensure = [&](unsigned need) {   // warp-uniform: descriptors of the tiles in `need`
    if (todo & need) {
      wait_len();
      if ((todo >> lane) & 1u) ring[lane] = make_meta(lane, (desc_mask >> lane) & 1u);
      todo = 0;
      __syncwarp();
    }
  };
  const unsigned first = (nt >= SPW ? (1u << SPW) - 1u : (1u << nt) - 1u) & ~pre_mask;
  ensure(first);
  if ((first >> lane) & 1)
    stg(smem + (warp * SPW + lane) * T::STAGE_BYTES, &full[warp * SPW + lane],
                  ring[lane], 0);

  // ================= tiles of this warp
  bool failed = false;
  int merge_h = -1;   // a shared head whose parts this warp merges
  for (int k = 0; k < nt; ++k) {
    const int s = warp * SPW + (k % SPW);
    ensure(k < 32 ? 1u << k : 0u);
    const TileMeta tm = ring[k % NMR];
    int h, lp;
    head_of(k, h, lp);
    if (!failed) {
      const bool ok = mbar_wait(&full[s], (k / SPW) & 1);
      if (!__all_sync(0xffffffffu, ok)) {
        // a copy did not land in time: latch the error, give the warp's other
        // stage in flight one more bounded wait so that no copy is left
        // pending into shared memory when the CTA leaves, and go on without
        // arithmetic, so that every head's partial count still completes
        if (lane == 0) {
          latch_error(c.ctr, FDMS_ERR_DEVICE);
          if (k + 1 < nt) mbar_wait(&full[warp * SPW + ((k + 1) % SPW)], ((k + 1) / SPW) & 1);
        }
        __syncwarp();
        failed = true;
      }
    }
    if (!failed) {
      // (only pending ring rows, which a tile described after the wait holds,
      // need the position count now)
      const int thresh = ((tm.rows >> 16) & kPending) ? cn[h] - c.W : 0;
      if (BLK && ((tm.rows >> 16) & kFirst)) {   // a head starts: both running states empty
        wt.reset();
        wt16.reset();
      }
      if (BLK && ((tm.rows >> 16) & kBf16)) {
        if (h != wt16.cur_hidx) wt16.fetch_q(q_of(h), h);
        wt16.tile(smem + s * T::STAGE_BYTES, tm, thresh, c.ring_keep + (hi0 + h) * c.Rpad, c.R,
                  lane);
      } else {
        if (h != wt.cur_hidx) wt.fetch_q(q_of(h), h);
        wt.tile(smem + s * T::STAGE_BYTES, tm, thresh, c.ring_keep + (hi0 + h) * c.Rpad, c.R,
                lane);
      }
      __syncwarp();
      // descriptors come HALF at a time: those of tiles k + HALF + 1 .. k + NMR
      // once tile k + 1 starts a new HALF
      if ((k + 1) % HALF == 0 && k + HALF + 1 < nt) {
        wait_len();
        fill(k + HALF + 1, HALF);
        __syncwarp();
      }
      // the stage is free: refill it with tile k + SPW
      ensure(k + SPW < 32 ? 1u << (k + SPW) : 0u);
      if (lane == 0 && k + SPW < nt)
        stg(smem + s * T::STAGE_BYTES, &full[s], ring[(k + SPW) % NMR], 0);
    } else if ((tm.rows >> 16) & kFirst) {
      wt.reset();   // an empty partial for the heads still to come
      if (BLK) wt16.reset();
    }

    // ---- end of this head inside the range
    if (!((tm.rows >> 16) & kLast)) continue;
    float o[MT][4], L0, L1;
    wt.finish(o, L0, L1);
    float vhead = hsc[2 * h + 1];
    if constexpr (BLK) {   // the bf16 tiles' partial joins, in the E4M3 layout and V unit 1
      float o16[MT][4], K0, K1;
      wt16.finish(o16, K0, K1);
      merge_kinds<MT>(o, wt.m0, wt.m1, L0, L1, vhead, o16, wt16.m0, wt16.m1, K0, K1, lane);
      vhead = 1.0f;
      if (k + 1 < nt) wt16.fetch_q(q_of(h + 1), h + 1);
    }
    if (k + 1 < nt) wt.fetch_q(q_of(h + 1), h + 1);   // the range's next head
    const int kb = h / c.Hkv, kh = h % c.Hkv;
    if (page_off[h] >= gp0 && page_off[h + 1] <= gp0 + nt) {
      // the whole head lies in this warp's range: write the output now
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hq = 2 * wt.t + e;
        if (hq >= G) continue;
        const float mh = e ? wt.m1 : wt.m0, lh = e ? L1 : L0;
        const float inv = mh == -INFINITY ? 0.f : vhead / lh;
        const long long ob = ((long long)kb * c.Hq + (long long)kh * G + hq) * D;
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const float ov = o[i][2 * hf + e] * inv;
            const long long oi = ob + T::vdim(i, wt.g, hf);
            if (oa.f32) static_cast<float*>(oa.out)[oi] = ov;
            else static_cast<uint16_t*>(oa.out)[oi] = f32_to_bf16_rn(ov);
          }
        if (oa.lse && wt.g == 0)
          oa.lse[(long long)kb * c.Hq + kh * G + hq] =
              mh == -INFINITY ? -INFINITY : (mh + log2f(lh)) * 0.6931471805599453f;
      }
      continue;
    }
    // shared with other warps: this warp's partial goes to the workspace at
    // v + h (unique: a warp's heads are consecutive, and later warps never go
    // back to earlier heads), then it is counted on the head's counter
    const long long part = v_range + h;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int hq = 2 * wt.t + e;
      if (hq >= G) continue;
      float* po = w.part_o + (part * G + hq) * D;
#pragma unroll
      for (int i = 0; i < MT; ++i) {
        po[T::vdim(i, wt.g, 0)] = o[i][e] * vhead;
        po[T::vdim(i, wt.g, 1)] = o[i][2 + e] * vhead;
      }
      if (wt.g == 0) {
        w.part_ml[(part * G + hq) * 2] = e ? wt.m1 : wt.m0;
        w.part_ml[(part * G + hq) * 2 + 1] = e ? L1 : L0;
      }
    }
    __syncwarp();
    // the range that holds the head's last tile merges the parts; the others
    // count theirs (release: the partial is visible to whoever sees the count)
    // and go on without waiting
    if ((page_off[h + 1] - 1) / S != v_range) {
      if (lane == 0) red_add_release(&w.head_cnt[h], 1);
    } else {
      merge_h = h;   // merged once this range is done, when the tile state is dead
    }
  }
  // ---- the merge of the head whose last tile this range holds (at most one:
  // it is the range's first head, shared with earlier ranges)
  if (merge_h >= 0) {
    const int h = merge_h;
    const long long r0 = page_off[h] / S, r1 = (page_off[h + 1] - 1) / S;
    // wait (bounded) for the other parts: their warps are of this kernel and
    // wait for nothing, so they finish
    int ok = 1;
    if (lane == 0) {
      const unsigned long long t0 = globaltimer();
      while (ld_acquire(&w.head_cnt[h]) < (int)(r1 - r0)) {
        if (globaltimer() - t0 > kWaitLimitNs) {
          ok = 0;
          latch_error(c.ctr, FDMS_ERR_DEVICE);
          break;
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);   // (a timed-out merge still reads only the workspace)
    __syncwarp();                            // after lane 0's acquire
    merge_parts<T>(c, w, oa, h, r0 + h, (int)(r1 - r0 + 1), lane);
    if (lane == 0) w.head_cnt[h] = 0;   // ready for the next call
  }

  // ---- this CTA's share of the snapshots the next decode of the layer plans
  // from (the other copy than the one this call read), and the counters
  wait_len();
  if (len_ok) {
    const int per = (NH + (int)gridDim.x - 1) / (int)gridDim.x;
    const int h0 = (int)blockIdx.x * per, h1 = min(NH, h0 + per);
    for (int h = h0 + tid; h < h1; h += NT) w.snap_wr[hi0 + h] = make_int4(cl[h], cn[h], cr[h], 0);
    if (blockIdx.x == 0) {
      unsigned long long slots = 0, bytes = 0;
      for (int h = tid; h < NH; h += NT) {
        slots += (unsigned long long)(cl[h] + (cn[h] - cr[h]));
        bytes += head_kv_bytes(c, cl[h], cn[h], cr[h]);
      }
      for (int off = 16; off > 0; off >>= 1) {
        slots += __shfl_xor_sync(0xffffffffu, slots, off);
        bytes += __shfl_xor_sync(0xffffffffu, bytes, off);
      }
      if (lane == 0 && slots) atomicAdd(&c.ctr->slots_decoded, slots);
      if (lane == 0 && bytes) atomicAdd(&c.ctr->bytes_decoded, bytes);
      if (tid == 0) atomicAdd(&c.ctr->decode_calls, 1ull);
    }
  }
}

// ------------------------------------------------------------------ dispatch
// Cluster size for a call of nh heads: the largest of 8, 4 and 2 at which
// every head gets its cluster at once on this device
// (cudaOccupancyMaxActiveClusters, queried at set-up: clusters live inside one
// GPC, so fewer fit than SMs / CS); 0 selects the global plan (more heads than
// that), which a cache created with an explicit split grid (decode_ctas > 0)
// always uses.
inline int cluster_size(const fdms_cache* cache, int nh) {
#if FDMS_CLUSTER_DECODE
  if (!cache->cluster_ok || cache->cfg.decode_ctas > 0) return 0;
  if (nh <= cache->max_clusters[3]) return 8;
  if (nh <= cache->max_clusters[2]) return 4;
  if (nh <= cache->max_clusters[1]) return 2;
#endif
  (void)cache;
  (void)nh;
  return 0;
}

template <class T, int CS, bool BLK>
cudaError_t launch_cluster_t(fdms_cache* cache, const DecodeWork& w, OutArgs oa, int layer,
                             int batch, const void* q, cudaStream_t s, int use_snap) {
  const int nh = batch * cache->view.Hkv;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nh * CS));
  cfg.blockDim = dim3(T::NT);
  cfg.dynamicSmemBytes = T::smem_bytes_cluster(cache->view.max_blocks);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = CS;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_decode_split<T, CS, BLK>, cache->view, w, oa, layer, batch,
                            static_cast<const uint16_t*>(q), use_snap);
}

// Snapshots may be used when the last decode of the layer (their writer) has
// certainly finished; the global plan also needs that decode to have covered
// every sequence of this call and few tokens appended since (its spares).
constexpr long long kSnapMaxTokens = 64;

template <class T>
fdms_status launch_split_t(fdms_cache* cache, const DecodeWork& w_in, OutArgs oa, int layer,
                           int batch, const void* q, cudaStream_t s) {
  const int nh = batch * cache->view.Hkv;
  // the snapshot copy this call reads, and the one it leaves for the next
  // decode of the layer
  const CacheView& cv = cache->view;
  const long long calls = cache->decode_count[layer];
  const size_t heads = (size_t)cv.L * cv.Bmax * cv.Hkv;
  DecodeWork w = w_in;
  w.snap_rd = w_in.snap + (size_t)(calls & 1) * heads;
  w.snap_wr = w_in.snap + (size_t)((calls + 1) & 1) * heads;
  const long long prev = cache->decode_at[layer];
  const bool writer_done = fdms_log_finished(cache, prev);
  const long long tokens = cache->tokens_since[layer];
  const int cs = cluster_size(cache, nh);
  cudaError_t e = cudaErrorUnknown;
  if (cs > 0) {
    const int use_snap = writer_done ? 1 : 0;
    if (T::FP8 && cache->view.blk)   // per-block FP8: two tile kinds
      e = cs == 8   ? launch_cluster_t<T, 8, T::FP8>(cache, w, oa, layer, batch, q, s, use_snap)
          : cs == 4 ? launch_cluster_t<T, 4, T::FP8>(cache, w, oa, layer, batch, q, s, use_snap)
                    : launch_cluster_t<T, 2, T::FP8>(cache, w, oa, layer, batch, q, s, use_snap);
    else
      e = cs == 8   ? launch_cluster_t<T, 8, false>(cache, w, oa, layer, batch, q, s, use_snap)
          : cs == 4 ? launch_cluster_t<T, 4, false>(cache, w, oa, layer, batch, q, s, use_snap)
                    : launch_cluster_t<T, 2, false>(cache, w, oa, layer, batch, q, s, use_snap);
    if (e != cudaSuccess) cudaGetLastError();   // a refused cluster launch falls back to the plan
  }
  if (e != cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cache->decode_ctas);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    bool done = false;
    if constexpr (T::FP8) {
      if (cache->view.blk) {
        // per-block FP8: two tile kinds per head, four warps per CTA (registers
        // for both running states), no snapshots (the staged block changes)
        constexpr int NWB = 4;
        using PL = PlanL<T, NWB>;
        cfg.blockDim = dim3(PL::NT);
        cfg.dynamicSmemBytes = PL::smem_bytes(nh);
        const int n_ranges = cache->decode_ctas * NWB;
        e = cudaLaunchKernelEx(&cfg, k_decode_plan<T, NWB, true>, cache->view, w, oa, layer,
                               batch, static_cast<const uint16_t*>(q), n_ranges,
                               1.0 / (double)n_ranges, 0, (int)tokens);
        done = true;
      }
    }
    if (!done) {
      constexpr int NW = PlanWarps<T>::value;
      using PL = PlanL<T, NW>;
      const int use_snap = prev > 0 && writer_done && batch <= cache->decode_batch[layer] &&
                                   tokens <= kSnapMaxTokens ? 1 : 0;
      cfg.blockDim = dim3(PL::NT);
      cfg.dynamicSmemBytes = PL::smem_bytes(nh);
      const int n_ranges = cache->decode_ctas * NW;
      e = cudaLaunchKernelEx(&cfg, k_decode_plan<T, NW, false>, cache->view, w, oa, layer, batch,
                             static_cast<const uint16_t*>(q), n_ranges, 1.0 / (double)n_ranges,
                             use_snap, (int)tokens);
    }
  }
  if (e != cudaSuccess) return FDMS_ERR_CUDA;
  const long long n = fdms_log_launch(cache, true);   // every decode kernel waits first
  cache->decode_at[layer] = n;
  cache->decode_batch[layer] = batch;
  cache->tokens_since[layer] = 0;
  cache->decode_count[layer] = calls + 1;
  return FDMS_OK;
}

template <class T, int CS>
int max_active_clusters(const fdms_cache* cache) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(CS * 64));
  cfg.blockDim = dim3(T::NT);
  cfg.dynamicSmemBytes = T::smem_bytes_cluster(cache->view.max_blocks);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  const int smem = (int)T::smem_bytes_cluster(cache->view.max_blocks);
  if (cudaFuncSetAttribute(k_decode_split<T, CS, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      (T::FP8 && cudaFuncSetAttribute(k_decode_split<T, CS, T::FP8>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      smem) != cudaSuccess) ||
      cudaOccupancyMaxActiveClusters(&n, k_decode_split<T, CS, false>, &cfg) != cudaSuccess)
    n = 0;
  return n;
}

template <class T>
fdms_status setup_t(fdms_cache* cache) {
  constexpr int NW = PlanWarps<T>::value;
  using PL = PlanL<T, NW>;
  const int nh = cache->view.Bmax * cache->view.Hkv;
  const size_t smem = PL::smem_bytes(nh);
  if (smem > 227 * 1024) return FDMS_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(k_decode_plan<T, NW, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return FDMS_ERR_UNSUPPORTED;
  if constexpr (T::FP8) {
    if (cache->view.blk) {   // the per-block FP8 variant (four warps)
      const size_t smem_b = PlanL<T, 4>::smem_bytes(nh);
      if (smem_b > 227 * 1024 ||
          cudaFuncSetAttribute(k_decode_plan<T, 4, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b) != cudaSuccess)
        return FDMS_ERR_UNSUPPORTED;
    }
  }
  // CTAs of the plan kernel resident per SM at the largest call (its merging
  // warps wait for the other parts of their head, so every CTA of a call must
  // be able to be resident at once)
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode_plan<T, NW, false>, PL::NT, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return FDMS_ERR_UNSUPPORTED;
  if constexpr (T::FP8) {
    if (cache->view.blk) {   // the per-block FP8 variant runs on the same grid
      int per_sm_b = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_b, k_decode_plan<T, 4, true>,
                                                        PlanL<T, 4>::NT,
                                                        PlanL<T, 4>::smem_bytes(nh)) !=
              cudaSuccess ||
          per_sm_b < 1)
        return FDMS_ERR_UNSUPPORTED;
      per_sm = std::min(per_sm, per_sm_b);
    }
  }
  cache->plan_ctas_per_sm = per_sm;
  cache->ctas_per_sm = per_sm;     // the plan fills every resident slot of the device
  cache->ranges_per_cta = NW;
  // per-head cluster mode: how many clusters of each size fit at once
  cache->max_clusters[0] = 0;
  cache->max_clusters[1] = max_active_clusters<T, 2>(cache);
  cache->max_clusters[2] = max_active_clusters<T, 4>(cache);
  cache->max_clusters[3] = max_active_clusters<T, 8>(cache);
  cache->cluster_ok = T::smem_bytes_cluster(cache->view.max_blocks) <= 227 * 1024 &&
                      cache->max_clusters[3] > 0;
  cudaGetLastError();   // a refused query only turns the cluster mode off
  return FDMS_OK;
}

template <int D, bool FP8, class F>
fdms_status by_group(int G, F&& f) {
  switch (G) {
    case 1: return f(Dec<D, FP8, 1>{});
    case 2: return f(Dec<D, FP8, 2>{});
    case 4: return f(Dec<D, FP8, 4>{});
    case 8: return f(Dec<D, FP8, 8>{});
  }
  return FDMS_ERR_UNSUPPORTED;
}

template <class F>
fdms_status by_config(const CacheView& c, F&& f) {
  if (c.D == 64 && !c.fp8) return by_group<64, false>(c.G, f);
  if (c.D == 64 && c.fp8) return by_group<64, true>(c.G, f);
  if (c.D == 128 && !c.fp8) return by_group<128, false>(c.G, f);
  if (c.D == 128 && c.fp8) return by_group<128, true>(c.G, f);
  return FDMS_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace fdms

using namespace fdms;

fdms_status fdms_decode_setup(fdms_cache* cache) {
  fdms_status st = by_config(cache->view, [&](auto t) { return setup_t<decltype(t)>(cache); });
  if (st != FDMS_OK) return st;
  // the plan's grid: every CTA that can be resident at once (more warps with
  // copies in flight: on a 253 MB call, 53 µs against 70 µs with one CTA per
  // SM); an explicit grid is capped at that
  const int resident = cache->num_sms * cache->plan_ctas_per_sm;
  const int ctas = cache->cfg.decode_ctas > 0 ? std::min(cache->cfg.decode_ctas, resident)
                                              : resident;
  cache->decode_ctas = ctas;
  const CacheView& c = cache->view;
  DecodeWork& w = cache->work;
  w.max_ctas = ctas;
  w.max_parts = ctas * cache->ranges_per_cta + c.Bmax * c.Hkv;   // range v, head h: v + h
  void* p = nullptr;
  auto take = [&](size_t bytes) -> void* {
    if (cudaMalloc(&p, bytes) != cudaSuccess || !fdms_track(cache, p, bytes)) return nullptr;
    if (cudaMemset(p, 0, bytes) != cudaSuccess) return nullptr;
    return p;
  };
  const size_t heads = (size_t)c.L * c.Bmax * c.Hkv;
  w.part_o = static_cast<float*>(take((size_t)w.max_parts * c.G * c.D * sizeof(float)));
  w.part_ml = static_cast<float*>(take((size_t)w.max_parts * c.G * 2 * sizeof(float)));
  w.snap = static_cast<int4*>(take(2 * heads * sizeof(int4)));
  w.snap_rd = w.snap_wr = nullptr;   // chosen per call
  w.head_cnt = static_cast<int*>(take((size_t)c.Bmax * c.Hkv * sizeof(int)));
  if (!w.part_o || !w.part_ml || !w.snap || !w.head_cnt) return FDMS_ERR_CUDA;
  return FDMS_OK;
}

fdms_status fdms_launch_decode(fdms_cache* cache, int layer, int batch, const void* q, void* out,
                               int out_f32, float* lse, cudaStream_t s) {
  OutArgs oa{out, lse, out_f32};
  return by_config(cache->view, [&](auto t) {
    return launch_split_t<decltype(t)>(cache, cache->work, oa, layer, batch, q, s);
  });
}

extern "C" fdms_status fdms_decode_layout(fdms_cache* cache, int batch, int* cluster_ctas_out,
                                          int* split_ctas_out) {
  if (!cache || batch < 1 || batch > cache->view.Bmax) return FDMS_ERR_INVALID_ARG;
  if (cluster_ctas_out) *cluster_ctas_out = cluster_size(cache, batch * cache->view.Hkv);
  if (split_ctas_out) *split_ctas_out = cache->decode_ctas;
  return FDMS_OK;
}

// ------------------------------------------------- decode without allocation
// A fixed scratch array for fdms_decode_attn_noalloc: the split partials and
// the merge counters of calls that run the global plan. Host code only learns
// its device address through cudaGetSymbolAddress (the host-side name is a
// stand-in, not a device pointer); device code never names it, it receives the
// address as arguments.
static __device__ __align__(256) unsigned char fdms_noalloc_scratch[FDMS_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(int device, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, fdms_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[device] = p;
  }
  *out = g_scratch_addr[device];
  return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" fdms_status fdms_decode_attn_noalloc(fdms_cache* cache, int layer, int batch,
                                                const void* q_dev, void* out_dev, void* stream) {
  if (!cache) return FDMS_ERR_INVALID_ARG;
  const CacheView& c = cache->view;
  if (layer < 0 || layer >= c.L || batch < 0 || batch > c.Bmax) return FDMS_ERR_INVALID_ARG;
  if (batch == 0) return FDMS_OK;
  if (!q_dev || !out_dev || (((uintptr_t)q_dev | (uintptr_t)out_dev) & 15))
    return FDMS_ERR_INVALID_ARG;
  if (cache->device < 0 || cache->device >= kMaxDevices) return FDMS_ERR_UNSUPPORTED;
  // layout of the scratch for this call: partials (o), partials (m, l), then
  // the merge counters (one per head of the call)
  const long long parts = (long long)cache->decode_ctas * cache->ranges_per_cta +
                          (long long)batch * c.Hkv;
  const size_t o_bytes = align256((size_t)parts * c.G * c.D * sizeof(float));
  const size_t ml_bytes = align256((size_t)parts * c.G * 2 * sizeof(float));
  const size_t cnt_bytes = align256((size_t)batch * c.Hkv * sizeof(int));
  const size_t need = o_bytes + ml_bytes + cnt_bytes;
  const bool plan = cluster_size(cache, batch * c.Hkv) == 0;
  // a call that runs in per-head clusters keeps its partials in shared memory
  if (plan && need > FDMS_STATIC_SCRATCH_BYTES) return FDMS_ERR_INVALID_ARG;

  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return FDMS_ERR_CUDA;
  if (prev != cache->device && cudaSetDevice(cache->device) != cudaSuccess) return FDMS_ERR_CUDA;
  void* base = nullptr;
  fdms_status st = FDMS_OK;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (scratch_address(cache->device, &base) != cudaSuccess) {
    st = FDMS_ERR_CUDA;
  } else {
    unsigned char* b = static_cast<unsigned char*>(base);
    DecodeWork w;
    w.part_o = reinterpret_cast<float*>(b);
    w.part_ml = reinterpret_cast<float*>(b + o_bytes);
    w.head_cnt = reinterpret_cast<int*>(b + o_bytes + ml_bytes);
    w.max_parts = (int)parts;
    w.max_ctas = cache->decode_ctas;
    w.snap = cache->work.snap;   // the cache's own memory, not scratch
    // the array keeps the previous call's contents: the merge counters must
    // start at zero, the partials are written before they are read
    if (plan && cudaMemsetAsync(w.head_cnt, 0, cnt_bytes, s) != cudaSuccess) st = FDMS_ERR_CUDA;
    OutArgs oa{out_dev, nullptr, 0};
    if (st == FDMS_OK)
      st = by_config(c, [&](auto t) {
        return launch_split_t<decltype(t)>(cache, w, oa, layer, batch, q_dev, s);
      });
  }
  if (prev != cache->device) cudaSetDevice(prev);
  return st;
}

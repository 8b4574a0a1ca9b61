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
//       thread-block cluster of 2-8 CTAs per pair; the head's tiles are split
//       over the cluster's warps in runs whose lengths differ by at most one;
//       the warps' partials (m, l, o) are merged in shared memory, the CTAs'
//       through distributed shared memory, and the cluster writes the output.
//       No plan, workspace or combine kernel.
//     * one plan (other calls): the tiles of all heads of the call are laid
//       end to end and cut into equal ranges, one per warp of the grid; heads
//       shared by several warps are merged by a combine kernel.
//   - The store is append-only and a ring slot keeps its row until the ring
//     wraps past it, so everything a decode call saw of a head stays where it
//     was. In cluster mode the call plans its tiles from what the previous
//     decode of the same layer saw (a per-head snapshot) and issues the copies
//     of those tiles before its dependency wait, while the kernel before it
//     still runs; after the wait it reads the head's current lengths, masks
//     ring rows that have been resolved since, extends the tiles at the end of
//     the store and of the ring, and adds tiles for what is new.
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

enum : int { kFirst = 1, kLast = 2, kRing = 4, kPending = 8 };

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
  static constexpr int Q_BYTES = G * D * 2;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES + ((Q_BYTES + 127) / 128) * 128;
  static constexpr int MK = TR / 16;           // 16-key row blocks per tile
  static constexpr int KS = D / 16;            // score k-steps (16 dims each)
  static constexpr int MT = D / 16;            // P.V row blocks (16 dims each)
  static constexpr bool PACK = G <= 4;         // p remainder in the spare MMA columns
  static_assert(TR >= 16 && TR <= 64 && 64 % TR == 0, "tiles tile a page");

  static constexpr int OFF_META = NSTAGE * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_META + NCW * NMR * (int)sizeof(TileMeta);
  static constexpr int OFF_HEADS = OFF_BAR + NSTAGE * 8;
  // global plan: head_off (i64), page_off (i32), len, n, r (i32), head scales (2 x f32)
  static size_t smem_bytes(int nh) {
    return 128 + OFF_HEADS + (size_t)(nh + 1) * 8 + (size_t)(nh + 1) * 4 +
           (size_t)nh * 4 * 3 + (size_t)nh * 8 + 64;
  }
  // per-head clusters: 16 ints of head state, then one slot of (o [G][D],
  // m [G], l [G]) per warp and one for the CTA
  static constexpr int SLOT = G * D + 2 * G;   // floats
  static constexpr int OFF_MERGE = OFF_HEADS + 64;
  static size_t smem_bytes_cluster() {
    return 128 + OFF_MERGE + (size_t)(NCW + 1) * SLOT * 4 + 64;
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
__device__ __forceinline__ int4 ld_dsmem_v4(uint32_t addr) {
  int4 v;
  asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
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
                                              float hs_k, float hs_v) {
  constexpr int TR = T::TR, RB = T::RB;
  TileMeta mt;
  mt.hidx = hidx;
  mt.pad = 0;
  int row0, row1, flags = 0;
  if (kind == 0) {
    const int j = idx * TR / kBlockSlots;
    row0 = 0;
    row1 = min(TR, len - idx * TR);
    const long long blk = c.block_table[hi * c.max_blocks + j];
    if (T::FP8) {
      mt.ks = c.bt_scale[(hi * c.max_blocks + j) * 2];
      mt.vrel = c.bt_scale[(hi * c.max_blocks + j) * 2 + 1] / hs_v;
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

// CS = 0: one plan over every head of the call, cut into equal tile ranges,
// partials merged by k_decode_combine. CS > 0 (calls with few heads): one
// cluster of CS CTAs per head, planned from the head's snapshot when use_snap
// (copies issued before the dependency wait); the cluster merges its warps'
// partials in shared memory and across CTAs through distributed shared memory
// and writes the output: no global plan, no workspace, no combine kernel.
template <class T, int CS>
__global__ void __launch_bounds__(T::NT, 1)
k_decode_split(CacheView c, DecodeWork w, OutArgs oa, int layer, int batch,
               const uint16_t* __restrict__ q, int n_ranges, double inv_ranges, int use_snap) {
  constexpr int D = T::D, G = T::G, RB = T::RB, TR = T::TR, SPW = T::SPW, MK = T::MK,
                KS = T::KS, MT = T::MT, NMR = T::NMR, NCW = T::NCW;
  constexpr bool FP8 = T::FP8, PACK = T::PACK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  const int NH = batch * c.Hkv;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long hi0 = (long long)layer * c.Bmax * c.Hkv;   // first head of this layer
  TileMeta* ring = reinterpret_cast<TileMeta*>(smem + T::OFF_META) + warp * NMR;

  // ---- set-up that reads no data the previous kernel writes: it overlaps
  // that kernel. Stale V rows of a stage are multiplied by p = 0, so they must
  // hold numbers: start from zeros, not from whatever bits shared memory held
  // (stale K rows only produce scores that are then masked).
  for (int i = tid; i < T::NSTAGE * (T::KV_BYTES / 16); i += T::NT) {
    const int st = i / (T::KV_BYTES / 16), off = i % (T::KV_BYTES / 16);
    reinterpret_cast<uint4*>(smem + st * T::STAGE_BYTES + T::KV_BYTES)[off] =
        make_uint4(0u, 0u, 0u, 0u);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // before any bulk copy
  if (lane < SPW) mbar_init(&full[warp * SPW + lane], 1);
  fence_mbar_init();

  // stage the K and V rows [row0, row1) of `mt` for tile k (one lane). phase 0:
  // the whole tile (arrive + K/V + q with a head's first tile); 1: K/V only, no
  // arrival (before the dependency wait); 2: the arrival and q of a tile whose
  // K/V phase 1 issued
  auto issue = [&](const TileMeta& mt, int k, int phase) {
    const int s = warp * SPW + k % SPW;
    uint8_t* kdst = smem + s * T::STAGE_BYTES;
    uint8_t* vdst = kdst + T::KV_BYTES;
    const int row0 = mt.rows & 0xFF, row1 = (mt.rows >> 8) & 0xFF;
    const uint32_t nb = row1 > row0 ? (uint32_t)(row1 - row0) * RB : 0u;
    const long long voff = (long long)((mt.rows >> 16) & kRing ? c.R : kBlockSlots) * RB;
    // q only with a warp's first tile of a head: the tiles after it keep the
    // head's q fragments in registers
    const bool with_q = ((mt.rows >> 16) & kFirst) != 0;
    const uint32_t qb = with_q ? (uint32_t)T::Q_BYTES : 0u;
    if (phase == 0) mbar_arrive_expect_tx(&full[s], 2u * nb + qb);
    if (phase == 1) mbar_expect_tx(&full[s], 2u * nb);
    if (phase == 2) mbar_arrive_expect_tx(&full[s], qb);
    if (phase != 2 && nb > 0) {
      bulk_g2s(kdst + row0 * RB, mt.ksrc + (long long)row0 * RB, nb, &full[s]);
      bulk_g2s(vdst + row0 * RB, mt.ksrc + voff + (long long)row0 * RB, nb, &full[s]);
    }
    if (with_q && phase != 1) {
      const int b = mt.hidx / c.Hkv, h = mt.hidx % c.Hkv;
      bulk_g2s(vdst + T::KV_BYTES, q + ((long long)b * c.Hq + (long long)h * G) * D,
               T::Q_BYTES, &full[s]);
    }
  };

  // ================================================= plan: this warp's tiles
  int nt = 0;                       // tiles of this warp
  unsigned pre_mask = 0;            // tiles k < SPW whose K/V went out before the wait
  TileMeta pre_mt;                  // lane k < SPW: what went out for tile k
  // cluster mode
  int* cst = reinterpret_cast<int*>(smem + T::OFF_HEADS);
  float* mslot = reinterpret_cast<float*>(smem + T::OFF_MERGE);
  const int hsel = CS > 0 ? (int)(blockIdx.x / (CS > 0 ? CS : 1)) : 0;
  const int crank = CS > 0 ? (int)(blockIdx.x % (CS > 0 ? CS : 1)) : 0;
  int sp_s = 0, f0_s = 0, a_first = 0, cnt = 0, e0 = 0, E_store = 0, fx0 = 0;
  // global plan
  long long* head_off = reinterpret_cast<long long*>(smem + T::OFF_HEADS);
  int* page_off = reinterpret_cast<int*>(head_off + NH + 1);
  int* s_len = page_off + NH + 1;
  int* s_n = s_len + NH;
  int* s_r = s_n + NH;
  float* s_hscale = reinterpret_cast<float*>(s_r + NH);
  int gp0 = 0, h_gs = 0, h_ge = 0;
  long long v_range = 0;

  if constexpr (CS > 0) {
    constexpr int NW = CS * NCW;              // warps of the cluster
    const int v = crank * NCW + warp;
    const long long hi = hi0 + hsel;
    // cst: [0..3] rank 0's copy of the snapshot, [4..6] snapshot planned on,
    // [8..10] lengths now, [12..13] FP8 head scales
    auto split = [&](int len_s, int n_s, int r_s) {
      sp_s = (len_s + TR - 1) / TR;
      f0_s = r_s / TR;
      const int P_s = head_tiles<TR>(len_s, n_s, r_s);
      const int qq = P_s / NW, rem = P_s % NW;
      cnt = qq + (v < rem ? 1 : 0);
      a_first = v * qq + min(v, rem);
      e0 = (v - rem + NW) % NW;               // extra tiles continue the round
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
      // ---- before the wait: the snapshot (one copy for the whole cluster)
      if (crank == 0 && tid == 0) {
        int4 sv = w.snap[hi];
        if (!(sv.x >= 0 && sv.x <= sv.z && sv.z <= sv.y && sv.y <= c.max_seq_len &&
              sv.y - sv.z <= c.R))
          sv = make_int4(0, 0, 0, 0);
        *reinterpret_cast<int4*>(cst) = sv;
      }
      cluster_sync_all();
      if (tid == 0) {
        const int4 sv = ld_dsmem_v4(cluster_addr(cst, 0));
        cst[4] = sv.x;
        cst[5] = sv.y;
        cst[6] = sv.z;
      }
      __syncthreads();
      const int len_s = cst[4], n_s = cst[5], r_s = cst[6];
      split(len_s, n_s, r_s);
      // the warp's first tiles, unless they can still grow (the last store
      // tile and the last ring frame when partly filled)
      const int k = lane;
      bool pre = false;
      if (k < SPW && k < cnt) {
        const int item = a_first + k;
        const int kind = item < sp_s ? 0 : 1;
        const int idx = kind == 0 ? item : f0_s + (item - sp_s);
        const bool edge = kind == 0 ? (idx == sp_s - 1 && len_s % TR != 0)
                                    : (idx == (n_s - 1) / TR && n_s % TR != 0);
        if (!edge) {
          pre_mt = tile_meta<T>(c, hi, hsel, kind, idx, len_s, n_s, r_s, 1.f, 1.f);
          pre_mt.rows |= (k == 0 ? kFirst : 0) << 16;
          issue(pre_mt, k, 1);
          pre = true;
        }
      }
      pre_mask = __ballot_sync(0xffffffffu, pre);
    }
    pdl_wait();                 // the previous kernel's writes are visible from here on
    pdl_launch_dependents();
    // the arrivals (and q, an input of this call) of the tiles issued early
    if ((pre_mask >> lane) & 1) issue(pre_mt, lane, 2);
    if (tid == 0) {
      const int len = c.store_len[hi], n = c.tok_n[hi], r = c.tok_r[hi];
      cst[8] = len;
      cst[9] = n;
      cst[10] = r;
      reinterpret_cast<float*>(cst)[12] = FP8 ? c.head_scale[hi * 2] : 1.0f;
      reinterpret_cast<float*>(cst)[13] = FP8 ? c.head_scale[hi * 2 + 1] : 1.0f;
      if (!use_snap) {
        cst[4] = len;
        cst[5] = n;
        cst[6] = r;
      }
      if (crank == 0) {
        if (w.snap) w.snap[hi] = make_int4(len, n, r, 0);
        atomicAdd(&c.ctr->slots_decoded, (unsigned long long)(len + (n - r)));
        if (blockIdx.x == 0) atomicAdd(&c.ctr->decode_calls, 1ull);
      }
    }
    __syncthreads();
    const int len_s = cst[4], n_s = cst[5], r_s = cst[6];
    const int len = cst[8], n = cst[9], r = cst[10];
    if (!use_snap) split(len_s, n_s, r_s);
    // tiles that are new since the snapshot: store tiles past its last one,
    // ring frames past its last one (and not below the current first)
    const int sp_c = (len + TR - 1) / TR;
    E_store = max(0, sp_c - sp_s);
    const int nfr_s = head_tiles<TR>(0, n_s, r_s);
    fx0 = max(nfr_s > 0 ? f0_s + nfr_s : r / TR, r / TR);
    const int E_ring = n > r ? max(0, (n - 1) / TR - fx0 + 1) : 0;
    const int E = E_store + E_ring;
    nt = cnt + (E > e0 ? (E - e0 + NW - 1) / NW : 0);
    if (lane < G) {   // an empty partial until the warp's last tile replaces it
      mslot[warp * T::SLOT + G * D + lane] = -INFINITY;
      mslot[warp * T::SLOT + G * D + G + lane] = 0.f;
    }
  } else {
    // warm L2 with this layer's lengths and block tables (read after the wait)
    {
      const long long bt_lines = ((long long)NH * c.max_blocks * 4 + 127) / 128;
      const char* btp = reinterpret_cast<const char*>(c.block_table + hi0 * c.max_blocks);
      for (long long i = (long long)blockIdx.x * T::NT + tid; i < bt_lines;
           i += (long long)gridDim.x * T::NT)
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
    pdl_wait();
    pdl_launch_dependents();
    // ---- units and pages of every head of the call; exclusive prefix
    const int per = (NH + T::NT - 1) / T::NT;
    const int h0 = tid * per, h1 = min(NH, h0 + per);
    long long su = 0;
    int sp = 0;
    for (int h = h0; h < h1; ++h) {
      const int len = c.store_len[hi0 + h], n = c.tok_n[hi0 + h], r = c.tok_r[hi0 + h];
      s_len[h] = len;
      s_n[h] = n;
      s_r[h] = r;
      s_hscale[2 * h] = FP8 ? c.head_scale[(hi0 + h) * 2] : 1.0f;
      s_hscale[2 * h + 1] = FP8 ? c.head_scale[(hi0 + h) * 2 + 1] : 1.0f;
      su += len + (n - r);
      sp += head_tiles<TR>(len, n, r);
    }
    long long iu = su;
    int ip = sp;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long au = __shfl_up_sync(0xffffffffu, iu, off);
      const int ap = __shfl_up_sync(0xffffffffu, ip, off);
      if (lane >= off) { iu += au; ip += ap; }
    }
    __shared__ long long s_wu[T::NT / 32];
    __shared__ int s_wp[T::NT / 32];
    if (lane == 31) { s_wu[warp] = iu; s_wp[warp] = ip; }
    __syncthreads();
    long long eu = iu - su;
    int ep = ip - sp;
    for (int i = 0; i < warp; ++i) { eu += s_wu[i]; ep += s_wp[i]; }
    for (int h = h0; h < h1; ++h) {
      head_off[h] = eu;
      page_off[h] = ep;
      eu += s_len[h] + (s_n[h] - s_r[h]);
      ep += head_tiles<TR>(s_len[h], s_n[h], s_r[h]);
    }
    if (tid == T::NT - 1) {
      head_off[NH] = eu;
      page_off[NH] = ep;
    }
    __syncthreads();
    const long long total = head_off[NH];
    const int P = page_off[NH];   // tiles of the call
    // Range v holds tiles [v S, (v + 1) S), S = ceil(P / ranges): a tile costs
    // the same compute full or not, so whole tiles are what gets balanced.
    const int S = tiles_per_warp(P, n_ranges, inv_ranges);
    if (blockIdx.x == 0 && tid == 0) {   // one thread, launches are ordered
      c.ctr->slots_decoded += (unsigned long long)total;
      c.ctr->decode_calls += 1ull;
    }
    // heads without a single slot get zeros (nobody else writes them)
    for (int h = blockIdx.x; h < NH; h += gridDim.x) {
      if (page_off[h + 1] != page_off[h]) continue;
      const int b = h / c.Hkv, kh = h % c.Hkv;
      for (int i = tid; i < G * D; i += T::NT) {
        const long long oi = ((long long)b * c.Hq + (long long)kh * G) * D + i;
        if (oa.f32) static_cast<float*>(oa.out)[oi] = 0.f;
        else static_cast<uint16_t*>(oa.out)[oi] = 0;
        if (oa.lse && i % D == 0) oa.lse[(long long)b * c.Hq + kh * G + i / D] = -INFINITY;
      }
    }
    // Range v goes to warp v / gridDim.x of CTA v % gridDim.x: when fewer
    // ranges than warps hold tiles, the busy ones are spread over every SM.
    v_range = (long long)warp * gridDim.x + blockIdx.x;
    if ((long long)blockIdx.x * S >= P) return;
    // ---- this warp's tiles [gp0, gp0 + nt) and the heads h_gs .. h_ge they
    // belong to (the number of heads h >= 1 with page_off[h] <= page)
    gp0 = (int)min(v_range * S, (long long)P);
    nt = min(gp0 + S, P) - gp0;
    if (nt > 0) {
      for (int base = 1; base < NH; base += 32) {
        const int h = base + lane;
        const int po = h < NH ? page_off[h] : P;
        h_gs += __popc(__ballot_sync(0xffffffffu, po <= gp0));
        h_ge += __popc(__ballot_sync(0xffffffffu, po <= gp0 + nt - 1));
      }
    }
  }

  // descriptor of this warp's tile k (one lane per tile), from the lengths now
  auto make_meta = [&](int k) -> TileMeta {
    TileMeta mt;
    if constexpr (CS > 0) {
      const int len = cst[8], n = cst[9], r = cst[10];
      int kind, idx;
      if (k < cnt) {
        const int item = a_first + k;
        kind = item < sp_s ? 0 : 1;
        idx = kind == 0 ? item : f0_s + (item - sp_s);
      } else {
        const int e = e0 + (k - cnt) * CS * NCW;
        kind = e < E_store ? 0 : 1;
        idx = kind == 0 ? sp_s + e : fx0 + (e - E_store);
      }
      const float* hs = reinterpret_cast<const float*>(cst) + 12;
      mt = tile_meta<T>(c, hi0 + hsel, hsel, kind, idx, len, n, r, hs[0], hs[1]);
      mt.rows |= ((k == 0 ? kFirst : 0) | (k == nt - 1 ? kLast : 0)) << 16;
    } else {
      const int gp = gp0 + k;
      // head of page gp: the last h in [h_gs, h_ge] with page_off[h] <= gp
      int h_lo = h_gs, h_hi = h_ge;
      while (h_lo < h_hi) {
        const int mid = (h_lo + h_hi + 1) >> 1;
        if (page_off[mid] <= gp) h_lo = mid; else h_hi = mid - 1;
      }
      const int hidx = h_lo;
      const int lp = gp - page_off[hidx];
      const int len = s_len[hidx], n = s_n[hidx], r = s_r[hidx];
      const int sp = (len + TR - 1) / TR;
      mt = tile_meta<T>(c, hi0 + hidx, hidx, lp < sp ? 0 : 1, lp < sp ? lp : r / TR + (lp - sp),
                        len, n, r, s_hscale[2 * hidx], s_hscale[2 * hidx + 1]);
      mt.rows |= ((k == 0 || lp == 0 ? kFirst : 0) |
                  (k == nt - 1 || gp + 1 == page_off[hidx + 1] ? kLast : 0)) << 16;
    }
    return mt;
  };
  // descriptors of tiles [k0, k0 + 32) into the warp's ring
  auto fill = [&](int k0) {
    const int k = k0 + lane;
    if (k < nt) ring[k % NMR] = make_meta(k);
  };
  fill(0);
  fill(32);
  __syncwarp();
  if (lane < SPW && lane < nt && !((pre_mask >> lane) & 1)) issue(ring[lane], lane, 0);


  // ================= tiles of this warp
  const int g = lane >> 2, t = lane & 3;
  const float qscale = c.softmax_scale * kLog2e;
  // P^T columns 2t and 2t + 1 of this lane: head, remainder or nothing
  const int role0 = PACK ? (2 * t < G ? 0 : (2 * t < 2 * G ? 1 : 2)) : 0;
  const int role1 = PACK ? (2 * t + 1 < G ? 0 : (2 * t + 1 < 2 * G ? 1 : 2)) : 0;
  const int qh = PACK ? g % G : g;   // query head of this lane's q column
  // This lane's row address for a matrix load: row 16 m + 8 ((lane >> 3) & 1) +
  // (lane & 7), chunk cb + (lane >> 4), so registers 0..3 receive the matrices
  // (rows 0-7, chunk cb), (rows 8-15, cb), (rows 0-7, cb + 1), (rows 8-15, cb + 1)
  // of row block m. Row blocks start at multiples of 8 rows, so the chunk
  // permutation of the row is that of lane & 7.
  const int lrow = 8 * ((lane >> 3) & 1) + (lane & 7);
  const int lsub = lane >> 4;
  const int lx = RB == 64 ? ((lane & 7) >> 1) & 3 : (lane & 7);
  auto lm_addr = [&](uint32_t base, int m, int cb) -> uint32_t {
    return base + (uint32_t)((16 * m + lrow) * RB + 16 * ((cb + lsub) ^ lx));
  };
  constexpr int NKL = FP8 ? KS / 2 : KS;   // K matrix loads per row block
  constexpr int NVL = FP8 ? MT / 2 : MT;   // V matrix loads per row block

  uint32_t qb[KS][2];          // q B-fragments (column g, k-steps)
  float qmul0 = 0.f, qmul1 = 0.f;   // score multipliers of columns 2t, 2t + 1
  int cur_hidx = -1;
  float m0 = -INFINITY, m1 = -INFINITY;   // running max of columns 2t, 2t + 1
  float l0 = 0.f, l1 = 0.f;               // this lane's part of their sums
  float oacc[MT][4];           // o^T: [dims of row block i] x [columns 2t, 2t + 1]
#pragma unroll
  for (int i = 0; i < MT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

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
    const int row0 = tm.rows & 0xFF, row1 = (tm.rows >> 8) & 0xFF, flags = tm.rows >> 16;
    const int hidx = tm.hidx;
    const uint8_t* Ks = smem + s * T::STAGE_BYTES;
    const uint8_t* Vs = Ks + T::KV_BYTES;
    const uint16_t* Qs = reinterpret_cast<const uint16_t*>(Vs + T::KV_BYTES);
    const uint32_t ks_base = smem_addr(Ks), vs_base = smem_addr(Vs);

    // ---- q fragments of the head (only when the head changes)
    if (hidx != cur_hidx) {
      cur_hidx = hidx;
      if constexpr (FP8) {
        // f16 q scaled by 2^a so that max |q| of the head is in [2^14, 2^15)
        // (bf16 -> f16 is then exact). K-slots 2t, 2t + 1, 2t + 8, 2t + 9 of
        // k-step s are dims 16 s + 4t .. 16 s + 4t + 3 (the order the E4M3 K
        // matrices give); the four lanes of a lane group hold a whole head.
        uint2 qw[KS];
        float amax = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          qw[s2] = *reinterpret_cast<const uint2*>(Qs + qh * D + 16 * s2 + 4 * t);
          amax = fmaxf(amax, fmaxf(fmaxf(fabsf(__uint_as_float(qw[s2].x << 16)),
                                         fabsf(__uint_as_float(qw[s2].x & 0xFFFF0000u))),
                                   fmaxf(fabsf(__uint_as_float(qw[s2].y << 16)),
                                         fabsf(__uint_as_float(qw[s2].y & 0xFFFF0000u)))));
        }
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
          qb[s2][0] = pack2<true>(__uint_as_float(qw[s2].x << 16) * up,
                                  __uint_as_float(qw[s2].x & 0xFFFF0000u) * up);
          qb[s2][1] = pack2<true>(__uint_as_float(qw[s2].y << 16) * up,
                                  __uint_as_float(qw[s2].y & 0xFFFF0000u) * up);
        }
        // column c carries query head c % G (c when G = 8); lane 4c holds its multiplier
        qmul0 = __shfl_sync(0xffffffffu, qm, 4 * (2 * t));
        qmul1 = __shfl_sync(0xffffffffu, qm, 4 * (2 * t + 1));
      } else {
        qmul0 = qmul1 = qscale;
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          qb[s2][0] = *reinterpret_cast<const uint32_t*>(Qs + qh * D + 16 * s2 + 2 * t);
          qb[s2][1] = *reinterpret_cast<const uint32_t*>(Qs + qh * D + 16 * s2 + 8 + 2 * t);
        }
      }
    }
    if (flags & kFirst) {
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
#pragma unroll
      for (int i = 0; i < MT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    }

    // ---- visible rows of the tile frame: [row0, row1), less the pending ring
    // rows whose keep bit is 0 (one ring_keep byte per row, read only then)
    const bool pend = (flags & kPending) != 0;
    const bool full_tile = row0 == 0 && row1 == TR && !pend;
    unsigned long long vmask = ~0ull;
    if (!full_tile) {
      vmask = (row1 >= 64 ? ~0ull : (1ull << row1) - 1ull) & ~((1ull << row0) - 1ull);
      if (pend) {
        const int thresh = (CS > 0 ? cst[9] : s_n[hidx]) - c.W;
        const long long keep_base = (hi0 + hidx) * c.Rpad;
#pragma unroll
        for (int h2 = 0; h2 < (TR + 31) / 32; ++h2) {
          const int row = 32 * h2 + lane;
          bool drop = false;
          if (row < TR && row >= row0 && row < row1) {
            const int p = tm.p0 + row;
            drop = p < thresh && c.ring_keep[keep_base + p % c.R] == 0;
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
    __syncwarp();
    // the stage is free: refill it with tile k + SPW (descriptors come 32 at a
    // time, those of tiles k + 33 .. k + 64 once tile k + 1 starts a new 32)
    if ((k + 1) % 32 == 0 && k + 33 < nt) {
      fill(k + 33);
      __syncwarp();
    }
    if (lane == 0 && k + SPW < nt) issue(ring[(k + SPW) % NMR], k + SPW, 0);

    // ---- end of this head inside the range
    if (flags & kLast) {
      float L0 = l0, L1 = l1;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        L0 += __shfl_xor_sync(0xffffffffu, L0, off);
        L1 += __shfl_xor_sync(0xffffffffu, L1, off);
      }
      // a head's p head and remainder columns summed: columns h and h + G
      float o[MT][4];
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
      float vhead;
      if constexpr (CS > 0) vhead = reinterpret_cast<const float*>(cst)[13];
      else vhead = s_hscale[2 * hidx + 1];
      const int kb = hidx / c.Hkv, kh = hidx % c.Hkv;
      // lane 4g + t holds heads 2t (element 0) and 2t + 1 (element 1)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = 2 * t + e;
        if (h >= G) continue;
        const float mh = e ? m1 : m0, lh = e ? L1 : L0;
        if constexpr (CS > 0) {   // the warp's partial, for the CTA's merge
          float* po = mslot + warp * T::SLOT;
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            po[h * D + T::vdim(i, g, 0)] = o[i][e] * vhead;
            po[h * D + T::vdim(i, g, 1)] = o[i][2 + e] * vhead;
          }
          if (g == 0) {
            po[G * D + h] = mh;
            po[G * D + G + h] = lh;
          }
        } else if (page_off[hidx] >= gp0 && page_off[hidx + 1] <= gp0 + nt) {
          // the whole head lies in this warp's range: write the output now
          const float inv = mh == -INFINITY ? 0.f : vhead / lh;
          const long long ob = ((long long)kb * c.Hq + (long long)kh * G + h) * D;
#pragma unroll
          for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const float ov = o[i][2 * hf + e] * inv;
              const long long oi = ob + T::vdim(i, g, hf);
              if (oa.f32) static_cast<float*>(oa.out)[oi] = ov;
              else static_cast<uint16_t*>(oa.out)[oi] = f32_to_bf16_rn(ov);
            }
          if (oa.lse && g == 0)
            oa.lse[(long long)kb * c.Hq + kh * G + h] =
                mh == -INFINITY ? -INFINITY : (mh + log2f(lh)) * 0.6931471805599453f;
        } else {
          // shared with other warps: this warp's partial goes to the workspace,
          // at v + hidx (unique: a warp's heads are consecutive, and later
          // warps never go back to earlier heads)
          const long long part = v_range + hidx;
          float* po = w.part_o + (part * G + h) * D;
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            po[T::vdim(i, g, 0)] = o[i][e] * vhead;
            po[T::vdim(i, g, 1)] = o[i][2 + e] * vhead;
          }
          if (g == 0) {
            w.part_ml[(part * G + h) * 2] = mh;
            w.part_ml[(part * G + h) * 2 + 1] = lh;
          }
        }
      }
    }
  }

  if constexpr (CS > 0) {
    // ---- merge: the warps' partials into the CTA's (shared memory), then the
    // CTAs' partials across the cluster; each CTA writes 1/CS of the head's
    // output. o = sum_w 2^(m_w - M) o_w / sum_w 2^(m_w - M) l_w.
    __syncthreads();
    float* cpart = mslot + NCW * T::SLOT;
    for (int e = tid; e < G * D; e += T::NT) {
      const int h = e / D;
      float mv[NCW], M = -INFINITY;
#pragma unroll
      for (int v = 0; v < NCW; ++v) {
        mv[v] = mslot[v * T::SLOT + G * D + h];
        M = fmaxf(M, mv[v]);
      }
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int v = 0; v < NCW; ++v) {
          if (mv[v] != -INFINITY) {   // empty partials hold no o values
            const float bw = fast_exp2(mv[v] - M);
            L += mslot[v * T::SLOT + G * D + G + h] * bw;
            O += mslot[v * T::SLOT + e] * bw;
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
}

// Merge of the warp partials of one (seq, kv head) that several warps covered:
// o = sum_w 2^(m_w - M) o_w / sum_w 2^(m_w - M) l_w. Heads inside one warp's
// range, or with no slot, were written by the split kernel. CPH CTAs share a
// head, TPE adjacent threads one output element: each loads its share of the
// partials (up to kChunk at once, all loads before any use), merges them, and
// the TPE results are merged across the threads by shuffles. Up to
// TPE * kChunk partials per head cost one round trip to memory.
template <int D, int G>
struct Combine {
  static constexpr int NE = G * D;    // output elements of a head
  static constexpr int TPE = 4;       // threads per element
  static constexpr int NT = 256;      // threads per CTA
  static constexpr int EPC = NT / TPE;                 // elements per CTA
  static constexpr int CPH = NE / EPC;                 // CTAs per head
  static_assert(NE % EPC == 0, "whole CTAs per head");
};

// merge (M2, L2, O2) into (M, L, O), both in the log2 domain
__device__ __forceinline__ void merge_mlo(float& M, float& L, float& O, float M2, float L2,
                                          float O2) {
  const float mx = fmaxf(M, M2);
  if (mx == -INFINITY) return;
  const float a = fast_exp2(M - mx), b = fast_exp2(M2 - mx);   // 0 for an empty side
  L = L * a + L2 * b;
  O = O * a + O2 * b;
  M = mx;
}

template <int D, int G, int TR>
__global__ void __launch_bounds__(Combine<D, G>::NT)
k_decode_combine(CacheView c, DecodeWork w, int layer, int batch, OutArgs oa, int n_ranges,
                 double inv_ranges) {
  using C = Combine<D, G>;
  constexpr int kChunk = 16, TPE = C::TPE;
  pdl_launch_dependents();
  const int hidx = blockIdx.x / C::CPH, tid = threadIdx.x, sub = tid % TPE;
  // ---- the split's plan, rebuilt before the wait: it depends only on the
  // head lengths, which no kernel between the split and this one changes (the
  // append that set them had finished before the split began)
  __shared__ int s_sum[C::NT / 32];
  __shared__ int s_head[2];   // tile prefix at hidx and hidx + 1
  __shared__ int s_total;
  {
    const int NH = batch * c.Hkv;
    const long long hi0 = (long long)layer * c.Bmax * c.Hkv;
    const int per = (NH + C::NT - 1) / C::NT;
    const int h0 = min(NH, tid * per), h1 = min(NH, h0 + per);
    int sp = 0, sp_at = 0, sp_next = 0;
    for (int h = h0; h < h1; ++h) {
      if (h == hidx) sp_at = sp;
      if (h == hidx + 1) sp_next = sp;
      sp += head_tiles<TR>(c.store_len[hi0 + h], c.tok_n[hi0 + h], c.tok_r[hi0 + h]);
    }
    const int lane = tid % 32, warp = tid / 32;
    int incl = sp;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) s_sum[warp] = incl;
    __syncthreads();
    int excl = incl - sp;
    for (int i = 0; i < warp; ++i) excl += s_sum[i];
    if (hidx >= h0 && hidx < h1) s_head[0] = excl + sp_at;
    if (hidx + 1 >= h0 && hidx + 1 < h1) s_head[1] = excl + sp_next;
    if (tid == C::NT - 1) s_total = excl + sp;
    __syncthreads();
    if (hidx + 1 == NH && tid == 0) s_head[1] = s_total;
    __syncthreads();
  }
  const int hs = s_head[0], he = s_head[1];
  const int S = tiles_per_warp(s_total, n_ranges, inv_ranges);
  pdl_wait();
  if (he == hs) return;
  const long long r0 = hs / S, r1 = (he - 1) / S;
  if (r0 == r1) return;
  const int Hkv = c.Hkv, Hq = c.Hq;
  const int kb = hidx / Hkv, kh = hidx % Hkv;
  const int idx = (blockIdx.x % C::CPH) * C::EPC + tid / TPE;
  const int h = idx / D, d = idx % D;
  float M = -INFINITY, L = 0.f, O = 0.f;
  for (long long p0 = r0 + sub; p0 <= r1; p0 += (long long)kChunk * TPE) {
    float mb[kChunk], lb[kChunk], ob[kChunk];
#pragma unroll
    for (int u = 0; u < kChunk; ++u) {   // loads first, all independent
      const long long pr = p0 + (long long)u * TPE;
      const long long pp = pr + hidx;
      const bool live = pr <= r1;
      mb[u] = live ? __ldcg(&w.part_ml[(pp * G + h) * 2]) : -INFINITY;
      lb[u] = live ? __ldcg(&w.part_ml[(pp * G + h) * 2 + 1]) : 0.f;
      ob[u] = live ? __ldcg(&w.part_o[(pp * G + h) * D + d]) : 0.f;
    }
    float mx = M;
#pragma unroll
    for (int u = 0; u < kChunk; ++u) mx = fmaxf(mx, mb[u]);
    if (mx == -INFINITY) continue;
    const float a = fast_exp2(M - mx);   // 0 while M is -inf
    L *= a;
    O *= a;
#pragma unroll
    for (int u = 0; u < kChunk; ++u) {
      const float bb = fast_exp2(mb[u] - mx);   // 0 for empty partials
      L += lb[u] * bb;
      O += ob[u] * bb;
    }
    M = mx;
  }
#pragma unroll
  for (int off = 1; off < TPE; off <<= 1)
    merge_mlo(M, L, O, __shfl_xor_sync(0xffffffffu, M, off),
              __shfl_xor_sync(0xffffffffu, L, off), __shfl_xor_sync(0xffffffffu, O, off));
  if (sub != 0) return;
  const float o = M == -INFINITY ? 0.f : O / L;
  const long long oi = ((long long)kb * Hq + (long long)kh * G + h) * D + d;
  if (oa.f32) static_cast<float*>(oa.out)[oi] = o;
  else static_cast<uint16_t*>(oa.out)[oi] = f32_to_bf16_rn(o);
  if (oa.lse && d == 0)
    oa.lse[(long long)kb * Hq + kh * G + h] =
        M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
}

// ------------------------------------------------------------------ dispatch
// Cluster size for a call of nh heads: the largest of 8, 4, 2 with nh clusters
// of that size resident at once on this device (cudaOccupancyMaxActiveClusters,
// queried at set-up: clusters live inside one GPC, so fewer fit than SMs / CS);
// 0 selects the global plan and the combine kernel, which a cache created with
// an explicit split grid (decode_ctas > 0) always uses.
inline int cluster_size(const fdms_cache* cache, int nh) {
#if FDMS_CLUSTER_DECODE
  if (!cache->cluster_ok || cache->cfg.decode_ctas > 0) return 0;
  for (int i = 3; i >= 1; --i)
    if (nh <= cache->max_clusters[i]) return 1 << i;
#endif
  (void)cache;
  (void)nh;
  return 0;
}

template <class T, int CS>
cudaError_t launch_cluster_t(fdms_cache* cache, const DecodeWork& w, OutArgs oa, int layer,
                             int batch, const void* q, cudaStream_t s) {
  const int nh = batch * cache->view.Hkv;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nh * CS));
  cfg.blockDim = dim3(T::NT);
  cfg.dynamicSmemBytes = T::smem_bytes_cluster();
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
  return cudaLaunchKernelEx(&cfg, k_decode_split<T, CS>, cache->view, w, oa, layer, batch,
                            static_cast<const uint16_t*>(q), 0, 0.0, w.snap ? 1 : 0);
}

template <class T>
fdms_status launch_split_t(fdms_cache* cache, const DecodeWork& w, OutArgs oa, int layer,
                           int batch, const void* q, cudaStream_t s) {
  const int nh = batch * cache->view.Hkv;
  const int cs = cluster_size(cache, nh);
  if (cs > 0) {
    const cudaError_t e = cs == 8   ? launch_cluster_t<T, 8>(cache, w, oa, layer, batch, q, s)
                          : cs == 4 ? launch_cluster_t<T, 4>(cache, w, oa, layer, batch, q, s)
                                    : launch_cluster_t<T, 2>(cache, w, oa, layer, batch, q, s);
    if (e == cudaSuccess) {
      cache->last_append_layer = -1;   // the kernel waits for every append queued before it
      return FDMS_OK;
    }
    cudaGetLastError();   // a refused cluster launch falls back to the global plan
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cache->decode_ctas);
  cfg.blockDim = dim3(T::NT);
  cfg.dynamicSmemBytes = T::smem_bytes(nh);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int n_ranges = cache->decode_ctas * T::NCW;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_decode_split<T, 0>, cache->view, w, oa, layer, batch,
                                     static_cast<const uint16_t*>(q), n_ranges,
                                     1.0 / (double)n_ranges, 0);
  if (e != cudaSuccess) return FDMS_ERR_CUDA;
  cache->last_append_layer = -1;   // the split waits for every append queued before it
  cfg.gridDim = dim3((unsigned)(nh * Combine<T::D, T::G>::CPH));
  cfg.blockDim = dim3(Combine<T::D, T::G>::NT);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, k_decode_combine<T::D, T::G, T::TR>, cache->view, w, layer, batch,
                         oa, n_ranges, 1.0 / (double)n_ranges);
  return e == cudaSuccess ? FDMS_OK : FDMS_ERR_CUDA;
}

template <class T, int CS>
int max_active_clusters() {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(CS * 64));
  cfg.blockDim = dim3(T::NT);
  cfg.dynamicSmemBytes = T::smem_bytes_cluster();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(k_decode_split<T, CS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)T::smem_bytes_cluster()) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, k_decode_split<T, CS>, &cfg) != cudaSuccess)
    n = 0;
  return n;
}

template <class T>
fdms_status setup_t(fdms_cache* cache) {
  const int nh = cache->view.Bmax * cache->view.Hkv;
  const size_t smem = T::smem_bytes(nh);
  if (smem > 227 * 1024) return FDMS_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(k_decode_split<T, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return FDMS_ERR_UNSUPPORTED;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode_split<T, 0>, T::NT,
                                                    smem) != cudaSuccess || per_sm < 1)
    return FDMS_ERR_UNSUPPORTED;
  cache->ctas_per_sm = per_sm;
  cache->ranges_per_cta = T::NCW;
  // per-head cluster mode: how many clusters of each size fit at once
  cache->max_clusters[0] = 0;
  cache->max_clusters[1] = max_active_clusters<T, 2>();
  cache->max_clusters[2] = max_active_clusters<T, 4>();
  cache->max_clusters[3] = max_active_clusters<T, 8>();
  cache->cluster_ok = T::smem_bytes_cluster() <= 227 * 1024 && cache->max_clusters[1] > 0;
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
  const int ctas = cache->cfg.decode_ctas > 0 ? cache->cfg.decode_ctas
                                              : cache->num_sms * cache->ctas_per_sm;
  cache->decode_ctas = ctas;
  const CacheView& c = cache->view;
  DecodeWork& w = cache->work;
  w.max_ctas = ctas;
  w.max_parts = ctas * cache->ranges_per_cta + c.Bmax * c.Hkv;   // range v, head h: v + h
  void* p = nullptr;
  auto take = [&](size_t bytes) -> void* {
    if (cudaMalloc(&p, bytes) != cudaSuccess || !fdms_track(cache, p, bytes)) return nullptr;
    return p;
  };
  const size_t heads = (size_t)c.L * c.Bmax * c.Hkv;
  w.part_o = static_cast<float*>(take((size_t)w.max_parts * c.G * c.D * sizeof(float)));
  w.part_ml = static_cast<float*>(take((size_t)w.max_parts * c.G * 2 * sizeof(float)));
  w.snap = static_cast<int4*>(take(heads * sizeof(int4)));
  if (!w.part_o || !w.part_ml || !w.snap) return FDMS_ERR_CUDA;
  if (cudaMemset(w.snap, 0, heads * sizeof(int4)) != cudaSuccess) return FDMS_ERR_CUDA;
  return FDMS_OK;
}

fdms_status fdms_launch_decode(fdms_cache* cache, int layer, int batch, const void* q, void* out,
                               int out_f32, float* lse, cudaStream_t s) {
  OutArgs oa{out, lse, out_f32};
  return by_config(cache->view, [&](auto t) {
    return launch_split_t<decltype(t)>(cache, cache->work, oa, layer, batch, q, s);
  });
}

// ------------------------------------------------- decode without allocation
// A fixed scratch array for fdms_decode_attn_noalloc: the split partials of
// calls that run the global plan. Host code only learns its device address
// through cudaGetSymbolAddress (the host-side name is a stand-in, not a device
// pointer); device code never names it, it receives the address as arguments.
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
  // layout of the scratch for this call: partials (o), then partials (m, l);
  // everything is written before it is read
  const long long parts = (long long)cache->decode_ctas * cache->ranges_per_cta +
                          (long long)batch * c.Hkv;
  const size_t o_bytes = align256((size_t)parts * c.G * c.D * sizeof(float));
  const size_t ml_bytes = align256((size_t)parts * c.G * 2 * sizeof(float));
  const size_t need = o_bytes + ml_bytes;
  // a call that runs in per-head clusters keeps its partials in shared memory
  if (cluster_size(cache, batch * c.Hkv) == 0 && need > FDMS_STATIC_SCRATCH_BYTES)
    return FDMS_ERR_INVALID_ARG;

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
    w.max_parts = (int)parts;
    w.max_ctas = cache->decode_ctas;
    w.snap = cache->work.snap;   // the cache's own memory, not scratch
    // the array keeps the previous call's contents; nothing in it needs to
    // start at zero (every value is written by this call before it is read)
    OutArgs oa{out_dev, nullptr, 0};
    st = by_config(c, [&](auto t) {
      return launch_split_t<decltype(t)>(cache, w, oa, layer, batch, q_dev, s);
    });
  }
  if (prev != cache->device) cudaSetDevice(prev);
  return st;
}

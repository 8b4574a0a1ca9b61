// Decode attention over the compact store: split kernel (+ combine kernel).
//
// FastDMS decodes over the survivors of per-head eviction only, reading 5-8x
// less KV than a dense cache ("FastDMS: 6.4X KV-cache compression running
// faster than vLLM BF16/FP8", aiwitness.kr/community/1t3vlrx, paragraph on
// decode speed and memory at 8K context). For query head g of kv head h:
//     o_g = sum_{j in S_h} softmax_j(scale * q_g . k_j) v_j,
// S_h = the head's compact store plus its visible ring slots.
//
// The kernel is memory bound: every byte of a visible K and V row is read once.
//   - Two ways to spread the work, chosen per call on the host:
//     * per-head clusters (calls with at most half as many heads as SMs): one
//       thread-block cluster of 2-8 CTAs per (seq, kv head); the head's tiles
//       (a tile = up to 32 rows of one 64-slot page for 128-byte rows: the
//       head's store pages, then its ring slots) are split evenly over the
//       cluster's CTAs and then their warps; the warps' partials (m, l, o) are
//       merged in shared memory, the CTAs' through distributed shared memory,
//       and the cluster writes the output. No plan, workspace or combine.
//     * one plan (other calls): the tiles of all heads of the call are laid
//       end to end and cut into equal ranges, one per warp of the grid; a warp
//       does the same number of tile steps whatever the mix of head lengths,
//       and emits one partial per head its range touches.
//   - Each warp stages its own tiles (32 rows of a 64-slot page for 128-byte
//     rows): the K rows, V rows and the head's q go to shared memory by 1-D
//     bulk copies (cp.async.bulk, completion on an mbarrier) into one of the
//     warp's two stages, and the warp refills a stage as soon as it has read
//     it. The tile descriptors (head, rows, source address) are worked out 32
//     at a time, one lane per tile, so the block-table reads of a warp's first
//     tiles overlap. Rows keep their page row in shared memory, so the chunk
//     permutation they are stored with makes the fragment loads below free of
//     bank conflicts.
//   - A warp computes the scores of a tile on the tensor cores
//     (mma.sync m16n8k16, fp32 accumulate; the G query heads of the kv head
//     are rows 0..G-1 of the 16-row A tile, keys are the columns), an online
//     softmax in fp32 in the log2 domain, and o^T += V^T p^T on the tensor
//     cores again (head dims are the rows, heads the columns, keys the
//     reduction): the score accumulators already have the layout of p^T's B
//     fragments. p is split into a 16-bit head and a 16-bit remainder so its
//     rounding stays below 2^-16 relative. FP8 pages are converted exactly to f16
//     (cvt e4m3x2 -> f16x2) and q is brought into f16 range by a power of two
//     that the score scale undoes; the page's K scale multiplies the scores
//     and its V scale the probabilities, never the elements.
//   - Plan mode: a head that lies whole inside one warp's range is written by
//     that warp; heads with no slot get zeros. Every other head has one partial
//     (m, l, o) per warp that covered part of it, written to a workspace; a
//     combine kernel merges them, four threads per output element, loading
//     all partials of the head at once:
//         o = sum_w 2^(m_w - M) o_w / sum_w 2^(m_w - M) l_w.
//     The combine rebuilds the split's tile plan from the head lengths itself
//     (nothing changes them between the two kernels), before its dependency
//     wait.
//   - Both kernels allow programmatic dependent launch: set-up that reads no
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
  const uint8_t* ksrc;   // first K row of the tile; its V rows follow the block's
                         // (or the ring's) K rows
  int hidx;              // head of the call (b * Hkv + h)
  int rows;              // row0 | row1 << 8 | flags << 16: frame rows [row0, row1)
  int p0;                // ring tiles: position of row row0
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
  static constexpr int NCW = G * D >= 1024 ? 4 : 8;   // warps (one unit range each)
  static constexpr int NT = NCW * 32;
  static constexpr int SPW = 2;                // stages per warp
  static constexpr int NSTAGE = NCW * SPW;
  static constexpr int NMR = 64;               // tile descriptors held per warp
  static constexpr int KV_BYTES = TR * RB;
  static constexpr int Q_BYTES = G * D * 2;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES + ((Q_BYTES + 127) / 128) * 128;
  static constexpr int NJ = TR / 8;            // score n-tiles (8 keys each)
  static constexpr int NU = TR / 16;           // p.v k-steps (16 keys each)
  static constexpr int KS = D / 16;            // q.k k-steps (16 dims each)
  static constexpr int MT = D / 16;            // p.v m-tiles (16 dims each)
  static constexpr int EC = 16 / ELT;          // elements per 16-byte chunk
  static constexpr int KCPT = RB / 64;         // K chunks per lane column (1, 2 or 4)
  static constexpr bool SPLIT = true;          // p = 16-bit head + 16-bit remainder
  static_assert(TR >= 16 && TR <= 64 && 64 % TR == 0, "tiles tile a page");

  static constexpr int OFF_META = NSTAGE * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_META + NCW * NMR * (int)sizeof(TileMeta);
  static constexpr int OFF_HEADS = OFF_BAR + NSTAGE * 8;
  static size_t smem_bytes(int nh) {
    // head_off (i64), page_off (i32), len, n, r (i32), head scales (2 x f32)
    return 128 + OFF_HEADS + (size_t)(nh + 1) * 8 + (size_t)(nh + 1) * 4 +
           (size_t)nh * 4 * 3 + (size_t)nh * 8 + 64;
  }
  // per-head (cluster) mode: a merge area after the head arrays, one slot of
  // (o [G][D], m [G], l [G]) per warp and one for the CTA
  static constexpr int SLOT = G * D + 2 * G;   // floats
  __host__ __device__ static size_t merge_off(int nh) {
    return ((size_t)OFF_HEADS + (size_t)(nh + 1) * 12 + (size_t)nh * 20 + 15) / 16 * 16;
  }
  static size_t smem_bytes_cluster(int nh) {
    return 128 + merge_off(nh) + (size_t)(NCW + 1) * SLOT * 4 + 64;
  }

  // unpermuted 16-byte K chunk i (0 .. KCPT-1) of lane column t
  __device__ static int kchunk(int t, int i) { return RB == 256 ? t + 4 * i : KCPT * t + i; }
  // element (dim) behind q.k k-step s, slot e (0..3) of lane column t:
  // e = 0, 1 are the fragment's k = 2t, 2t+1; e = 2, 3 are k = 2t+8, 2t+9
  __device__ static int kdim(int t, int s, int e) {
    const int se = 4 * s + e;
    return kchunk(t, se / EC) * EC + se % EC;
  }
  // dim of row g (hi = 0) or row g + 8 (hi = 1) of p.v m-tile i
  __device__ static int vdim(int g, int i, int hi) {
    if (RB == 256) return (i < 4 ? 8 * g + 2 * i : 64 + 8 * g + 2 * (i - 4)) + hi;
    return (D / 8) * g + 2 * i + hi;
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
// TR-row frames its ring slots r .. n-1 fall in.
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
// fp32 at the same shared-memory offset as `local` in CTA `rank` of the cluster
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
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

// CS = 0: one plan over every head of the call, cut into equal tile ranges,
// partials merged by k_decode_combine. CS > 0 (calls with few heads): one
// cluster of CS CTAs per head; the CTAs split the head's tiles, each merges its
// warps' partials in shared memory, and the cluster merges the CTAs' partials
// through distributed shared memory and writes the output: no global plan, no
// workspace, no combine kernel.
template <class T, int CS>
__global__ void __launch_bounds__(T::NT, 1)
k_decode_split(CacheView c, DecodeWork w, OutArgs oa, int layer, int batch,
               const uint16_t* __restrict__ q, int n_ranges, double inv_ranges) {
  constexpr int D = T::D, G = T::G, RB = T::RB, TR = T::TR, NSTAGE = T::NSTAGE,
                SPW = T::SPW, NJ = T::NJ, NU = T::NU, KS = T::KS, MT = T::MT, NMR = T::NMR;
  constexpr bool FP8 = T::FP8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  const int NH = batch * c.Hkv;
  long long* head_off = reinterpret_cast<long long*>(smem + T::OFF_HEADS);   // [NH + 1]
  int* page_off = reinterpret_cast<int*>(head_off + NH + 1);                 // [NH + 1]
  int* s_len = page_off + NH + 1;
  int* s_n = s_len + NH;
  int* s_r = s_n + NH;
  float* s_hscale = reinterpret_cast<float*>(s_r + NH);                      // [NH][2]

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long hi0 = (long long)layer * c.Bmax * c.Hkv;   // first head of this layer
  TileMeta* ring = reinterpret_cast<TileMeta*>(smem + T::OFF_META) + warp * NMR;

  // ---- set-up that reads no data the previous kernel writes: it overlaps
  // that kernel. Stale V rows of a stage are multiplied by p = 0, so they must
  // hold numbers: start from zeros, not from whatever bits shared memory held
  // (stale K rows only produce scores that are then masked).
  for (int i = tid; i < NSTAGE * (T::KV_BYTES / 16); i += T::NT) {
    const int st = i / (T::KV_BYTES / 16), off = i % (T::KV_BYTES / 16);
    reinterpret_cast<uint4*>(smem + st * T::STAGE_BYTES + T::KV_BYTES)[off] =
        make_uint4(0u, 0u, 0u, 0u);
  }
  // warm L2 with this layer's lengths and block tables (read after the wait)
  {
    const int NHL = batch * c.Hkv;
    const long long bt_lines = ((long long)NHL * c.max_blocks * 4 + 127) / 128;
    const char* btp = reinterpret_cast<const char*>(c.block_table + hi0 * c.max_blocks);
    for (long long i = (long long)blockIdx.x * T::NT + tid; i < bt_lines;
         i += (long long)gridDim.x * T::NT)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(btp + i * 128));
    if (tid < 4 && blockIdx.x < 8) {
      const char* arr = tid == 0   ? reinterpret_cast<const char*>(c.store_len + hi0)
                        : tid == 1 ? reinterpret_cast<const char*>(c.tok_n + hi0)
                        : tid == 2 ? reinterpret_cast<const char*>(c.tok_r + hi0)
                                   : reinterpret_cast<const char*>(c.head_scale + hi0 * 2);
      const int bytes = tid == 3 ? NHL * 8 : NHL * 4;   // this layer's slice only
      for (int j = blockIdx.x; j * 128 < bytes; j += 8)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(arr + j * 128));
    }
  }
  if (lane < SPW) mbar_init(&full[warp * SPW + lane], 1);
  fence_mbar_init();
  pdl_wait();                 // the previous kernel's writes are visible from here on
  pdl_launch_dependents();

  // ---- units and pages of every head of the call; exclusive prefix
  // cluster mode: the head of this CTA's cluster
  const int hsel = CS > 0 ? (int)(blockIdx.x / (CS > 0 ? CS : 1)) : 0;
  if constexpr (CS > 0) {
    if (tid == 0) {
      const long long hi = hi0 + hsel;
      const int len = c.store_len[hi], n = c.tok_n[hi], r = c.tok_r[hi];
      s_len[hsel] = len;
      s_n[hsel] = n;
      s_r[hsel] = r;
      s_hscale[2 * hsel] = FP8 ? c.head_scale[hi * 2] : 1.0f;
      s_hscale[2 * hsel + 1] = FP8 ? c.head_scale[hi * 2 + 1] : 1.0f;
      head_off[hsel] = 0;
      head_off[hsel + 1] = len + (n - r);
      page_off[hsel] = 0;
      page_off[hsel + 1] = head_tiles<TR>(len, n, r);
    }
    __syncthreads();
  } else {
    const int per = (NH + T::NT - 1) / T::NT;
    const int h0 = tid * per, h1 = min(NH, h0 + per);
    long long su = 0;
    int sp = 0;
    auto pages = [](int len, int live, int r) { return head_tiles<TR>(len, r + live, r); };
    for (int h = h0; h < h1; ++h) {
      const int len = c.store_len[hi0 + h], n = c.tok_n[hi0 + h], r = c.tok_r[hi0 + h];
      s_len[h] = len;
      s_n[h] = n;
      s_r[h] = r;
      s_hscale[2 * h] = FP8 ? c.head_scale[(hi0 + h) * 2] : 1.0f;
      s_hscale[2 * h + 1] = FP8 ? c.head_scale[(hi0 + h) * 2 + 1] : 1.0f;
      su += len + (n - r);
      sp += pages(len, n - r, r);
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
      ep += pages(s_len[h], s_n[h] - s_r[h], s_r[h]);
    }
    if (tid == T::NT - 1) {
      head_off[NH] = eu;
      page_off[NH] = ep;
    }
    __syncthreads();
  }
  int gp0 = 0, nt = 0, h_gs = 0, h_ge = 0;
  long long v_range = 0;
  float* mslot = reinterpret_cast<float*>(smem + T::merge_off(NH));   // cluster mode
  if constexpr (CS > 0) {
    // the head's tiles, split evenly over the cluster's CTAs, then over warps
    const int P = page_off[hsel + 1];
    const int crank = (int)(blockIdx.x % CS);
    const int per_c = (P + CS - 1) / CS;
    const int c0 = min(P, crank * per_c), c1 = min(P, c0 + per_c);
    const int per_w = (c1 - c0 + T::NCW - 1) / T::NCW;
    gp0 = min(c1, c0 + warp * per_w);
    nt = min(c1, gp0 + per_w) - gp0;
    h_gs = h_ge = hsel;
    if (crank == 0 && tid == 0) {
      atomicAdd(&c.ctr->slots_decoded, (unsigned long long)head_off[hsel + 1]);
      if (blockIdx.x == 0) atomicAdd(&c.ctr->decode_calls, 1ull);
    }
    if (lane < G) {   // an empty partial until the warp's last tile replaces it
      mslot[warp * T::SLOT + G * D + lane] = -INFINITY;
      mslot[warp * T::SLOT + G * D + G + lane] = 0.f;
    }
  } else {
  const long long total = head_off[NH];
  const int P = page_off[NH];   // tiles of the call
  // Range v holds tiles [v S, (v + 1) S), S = ceil(P / ranges): a tile costs
  // the same compute full or not, so whole tiles are what gets balanced. The
  // quotient is an fp64 estimate made exact by integer correction.
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

  // descriptor of this warp's tile k (one lane per tile)
  auto make_meta = [&](int k) -> TileMeta {
    TileMeta mt;
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
    const long long hi = hi0 + hidx;
    int flags = (k == 0 || lp == 0 ? kFirst : 0) |
                (k == nt - 1 || gp + 1 == page_off[hidx + 1] ? kLast : 0);
    int row0, row1;
    mt.hidx = hidx;
    mt.p0 = 0;
    mt.pad = 0;
    if (lp < sp) {   // store tile lp: block lp * TR / 64, rows from (lp * TR) % 64
      const int j = lp * TR / kBlockSlots;
      const int rb = (lp * TR) % kBlockSlots;          // block row of frame row 0
      row0 = 0;
      row1 = min(TR, len - lp * TR);
      const long long blk = c.block_table[hi * c.max_blocks + j];
      if (FP8) {
        mt.ks = c.bt_scale[(hi * c.max_blocks + j) * 2];
        mt.vrel = c.bt_scale[(hi * c.max_blocks + j) * 2 + 1] / s_hscale[2 * hidx + 1];
      } else {
        mt.ks = mt.vrel = 1.0f;
      }
      mt.ksrc = block_k(c, blk) + (long long)rb * RB;
    } else {         // ring tile: live units [TR*rp - off, TR*(rp+1) - off)
      const int rp = lp - sp, off = r % TR, live = n - r;
      const int a = max(TR * rp - off, 0), b = min(TR * (rp + 1) - off, live);
      const int p0 = r + a;
      const int slot0 = p0 % c.R;
      row0 = slot0 % TR;
      row1 = row0 + (b - a);
      mt.p0 = p0;
      flags |= kRing | (p0 < n - c.W ? kPending : 0);
      mt.ks = s_hscale[2 * hidx];
      mt.vrel = 1.0f;
      mt.ksrc = ring_k(c, hi) + (long long)slot0 * RB;
    }
    mt.rows = row0 | row1 << 8 | flags << 16;
    return mt;
  };
  // stage the K rows, V rows and q of tile k (one lane)
  auto issue = [&](const TileMeta& mt, int k) {
    const int s = warp * SPW + k % SPW;
    uint8_t* kdst = smem + s * T::STAGE_BYTES;
    uint8_t* vdst = kdst + T::KV_BYTES;
    const int row0 = mt.rows & 0xFF, row1 = (mt.rows >> 8) & 0xFF;
    const uint32_t nb = (uint32_t)(row1 - row0) * RB;
    const long long voff =
        (long long)((mt.rows >> 16) & kRing ? c.R : kBlockSlots) * RB;
    // q only with a warp's first tile of a head: the tiles after it keep the
    // head's q fragments in registers (each bulk copy costs issue time)
    const bool with_q = ((mt.rows >> 16) & kFirst) != 0;
    mbar_arrive_expect_tx(&full[s], 2u * nb + (with_q ? (uint32_t)T::Q_BYTES : 0u));
    bulk_g2s(kdst + row0 * RB, mt.ksrc, nb, &full[s]);
    bulk_g2s(vdst + row0 * RB, mt.ksrc + voff, nb, &full[s]);
    if (with_q) {
      const int b = mt.hidx / c.Hkv, h = mt.hidx % c.Hkv;
      bulk_g2s(vdst + T::KV_BYTES, q + ((long long)b * c.Hq + (long long)h * G) * D,
               T::Q_BYTES, &full[s]);
    }
  };
  // descriptors of tiles [k0, k0 + 32) into the warp's ring
  auto fill = [&](int k0) {
    const int k = k0 + lane;
    if (k < nt) ring[k % NMR] = make_meta(k);
  };
  // first descriptors; lanes 0 .. SPW-1 stage their tiles at once
  {
    const int k = lane;
    if (k < nt) {
      const TileMeta mt = make_meta(k);
      ring[k] = mt;
      if (k < SPW) issue(mt, k);
    }
    fill(32);
    __syncwarp();
  }

  // ================= tiles of this warp
  const int g = lane >> 2, t = lane & 3;
  const float qscale = c.softmax_scale * kLog2e;

  // shared-memory byte offsets of this lane's fragment loads inside a tile:
  // K rows 8j + g (the row permutation bits are g for every j), V rows
  // 16u + 2t + {0, 1, 8, 9} (permutation bits 2t + {0, 1})
  int koff[T::KCPT];
#pragma unroll
  for (int i = 0; i < T::KCPT; ++i)
    koff[i] = g * RB + 16 * swz_chunk(RB, false, g, T::kchunk(t, i));
  constexpr int VCHK = RB == 256 ? 2 : 1;
  int voff[4][VCHK];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const int rr = 2 * t + (q4 & 1) + 8 * (q4 >> 1);
#pragma unroll
    for (int ci = 0; ci < VCHK; ++ci)
      voff[q4][ci] = rr * RB + (RB == 64 ? 8 * g
                                          : 16 * swz_chunk(RB, true, rr, RB == 256 ? g + 8 * ci : g));
  }

  uint32_t qa[KS][2];          // q A-fragments (row g, k-steps)
  float qmul = 0.f;            // score multiplier of row g (scale, log2 e, q's power of two)
  int cur_hidx = -1;
  float m_run = -INFINITY, l_run = 0.f;    // softmax state of head g (shared by its quad)
  float oacc[MT][4];           // o^T: [dims g, g+8 of m-tile i] x [heads 2t, 2t+1]
#pragma unroll
  for (int i = 0; i < MT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

  for (int k = 0; k < nt; ++k) {
    const int s = warp * SPW + (k % SPW);
    const bool ok = mbar_wait(&full[s], (k / SPW) & 1);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
      break;
    }
    const TileMeta tm = ring[k % NMR];
    struct {
      int hidx, row0, row1, flags, p0, thresh, R;
      float ks, vrel, vhead;
      long long keep_base;
    } mt;
    mt.hidx = tm.hidx;
    mt.row0 = tm.rows & 0xFF;
    mt.row1 = (tm.rows >> 8) & 0xFF;
    mt.flags = tm.rows >> 16;
    mt.p0 = tm.p0;
    mt.thresh = s_n[tm.hidx] - c.W;
    mt.R = c.R;
    mt.ks = tm.ks;
    mt.vrel = tm.vrel;
    mt.vhead = s_hscale[2 * tm.hidx + 1];
    mt.keep_base = (hi0 + tm.hidx) * c.Rpad;
    const uint8_t* Ks = smem + s * T::STAGE_BYTES;
    const uint8_t* Vs = Ks + T::KV_BYTES;
    const uint16_t* Qs = reinterpret_cast<const uint16_t*>(Vs + T::KV_BYTES);
    const int row0 = mt.row0, row1 = mt.row1;

    // ---- q fragments of the head (only when the head changes)
    if (mt.hidx != cur_hidx) {
      cur_hidx = mt.hidx;
      if constexpr (FP8) {
        // f16 q scaled by 2^a so that max |q| of the row is in [2^14, 2^15)
        // (bf16 -> f16 is then exact). The 4 KS dims of lane column t are one
        // run of the row (the K chunks of the column are adjacent): 16-byte loads.
        constexpr int NQ = 4 * KS;   // q values of this lane
        static_assert(RB <= 128 && NQ == T::KCPT * T::EC, "one run of adjacent K chunks");
        uint32_t qw[NQ / 2];          // bf16 pairs, in k-slot order
        if (g < G) {
          const uint4* src = reinterpret_cast<const uint4*>(Qs + g * D + NQ * t);
#pragma unroll
          for (int i = 0; i < NQ / 8; ++i) {
            const uint4 x = src[i];
            qw[4 * i] = x.x; qw[4 * i + 1] = x.y; qw[4 * i + 2] = x.z; qw[4 * i + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < NQ / 2; ++i) qw[i] = 0u;
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < NQ / 2; ++i)
          amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(qw[i] << 16)),
                                   fabsf(__uint_as_float(qw[i] & 0xFFFF0000u))));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        int ex = 0;
        if (amax > 0.f) ex = 141 - (int)((__float_as_uint(amax) >> 23) & 0xFF);
        ex = max(-126, min(126, ex));
        const float up = __uint_as_float((uint32_t)(ex + 127) << 23);
        const float down = __uint_as_float((uint32_t)(127 - ex) << 23);
        qmul = qscale * down;
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          qa[s2][0] = pack2<true>(__uint_as_float(qw[2 * s2] << 16) * up,
                                  __uint_as_float(qw[2 * s2] & 0xFFFF0000u) * up);
          qa[s2][1] = pack2<true>(__uint_as_float(qw[2 * s2 + 1] << 16) * up,
                                  __uint_as_float(qw[2 * s2 + 1] & 0xFFFF0000u) * up);
        }
      } else {
        qmul = qscale;
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          const int d0 = T::kdim(t, s2, 0), d2 = T::kdim(t, s2, 2);
          qa[s2][0] = g < G ? *reinterpret_cast<const uint32_t*>(Qs + g * D + d0) : 0u;
          qa[s2][1] = g < G ? *reinterpret_cast<const uint32_t*>(Qs + g * D + d2) : 0u;
        }
      }
    }
    if (mt.flags & kFirst) {
      m_run = -INFINITY;
      l_run = 0.f;
#pragma unroll
      for (int i = 0; i < MT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    }

    // ---- visible rows of the tile frame: [row0, row1), less the pending ring
    // rows whose keep bit is 0 (one ring_keep byte per row, read only then)
    const bool pend = (mt.flags & kPending) != 0;
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
            const int p = mt.p0 + (row - row0);
            drop = p < mt.thresh && c.ring_keep[mt.keep_base + p % mt.R] == 0;
          }
          const unsigned bd = __ballot_sync(0xffffffffu, drop);
          vmask &= ~((unsigned long long)bd << (32 * h2));
        }
      }
      vmask >>= 2 * t;   // bit 8j + e: row 8j + 2t + e of this lane
    }

    // ---- scores of rows 8j + (0..7): S[head g][keys 8j + 2t, 8j + 2t + 1]
    float sc[NJ][2];
    const float mul = qmul * mt.ks;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t kw[T::KCPT][4];   // key row 8j + g, this lane's chunks
#pragma unroll
      for (int i = 0; i < T::KCPT; ++i) {
        const uint4 x = *reinterpret_cast<const uint4*>(Ks + 8 * j * RB + koff[i]);
        kw[i][0] = x.x; kw[i][1] = x.y; kw[i][2] = x.z; kw[i][3] = x.w;
      }
#pragma unroll
      for (int s2 = 0; s2 < KS; ++s2) {
        uint32_t b0, b1;
        if constexpr (FP8) {
          const uint32_t wv = kw[(4 * s2) / 16][((4 * s2) % 16) / 4];   // 4 codes
          b0 = e4m3x2_to_f16x2(wv & 0xFFFF);
          b1 = e4m3x2_to_f16x2(wv >> 16);
        } else {
          const int se = 4 * s2;                      // span elements 4 s2 .. 4 s2 + 3
          b0 = kw[se / 8][(se % 8) / 2];
          b1 = kw[se / 8][(se % 8) / 2 + 1];
        }
        mma16816<FP8>(acc, qa[s2][0], 0u, qa[s2][1], 0u, b0, b1);
      }
      sc[j][0] = acc[0] * mul;
      sc[j][1] = acc[1] * mul;
    }
    if (!full_tile) {
#pragma unroll
      for (int j = 0; j < NJ; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if (!((vmask >> (8 * j + e)) & 1ull)) sc[j][e] = -INFINITY;
    }

    // ---- online softmax for row (head) g; the 4 lanes of a quad share it.
    // With no visible key so far the reference point is 0: every p is then
    // 2^-inf = 0 and so is the rescale of the (empty) accumulators.
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < NJ; ++j) mx = fmaxf(mx, fmaxf(sc[j][0], sc[j][1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mn = fmaxf(m_run, mx);
    const float mref = mn == -INFINITY ? 0.f : mn;
    const float alpha = fast_exp2(m_run - mref);
    float pr[NJ][2];
    float ls = 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      pr[j][0] = fast_exp2(sc[j][0] - mref);
      pr[j][1] = fast_exp2(sc[j][1] - mref);
      ls += pr[j][0] + pr[j][1];
    }
    l_run = l_run * alpha + ls;
    m_run = mn;
    // o^T columns are heads 2t, 2t+1: their rescale factors live in quads 2t, 2t+1
    const float al_e = __shfl_sync(0xffffffffu, alpha, 8 * t);
    const float al_o = __shfl_sync(0xffffffffu, alpha, 8 * t + 4);
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      oacc[i][0] *= al_e;
      oacc[i][1] *= al_o;
      oacc[i][2] *= al_e;
      oacc[i][3] *= al_o;
    }

    // ---- o^T += V^T p^T, keys 16u .. 16u + 15 per k-step
#pragma unroll
    for (int u = 0; u < NU; ++u) {
      // p^T B fragment: (keys 16u + 2t, +1) and (16u + 8 + 2t, +1) of head g
      const float p0 = pr[2 * u][0] * mt.vrel, p1 = pr[2 * u][1] * mt.vrel;
      const float p2 = pr[2 * u + 1][0] * mt.vrel, p3 = pr[2 * u + 1][1] * mt.vrel;
      const uint32_t bh0 = pack2<FP8>(p0, p1), bh1 = pack2<FP8>(p2, p3);
      uint32_t bl0 = 0u, bl1 = 0u;
      if constexpr (T::SPLIT) {
        const float2 f0 = unpack2<FP8>(bh0), f1 = unpack2<FP8>(bh1);
        bl0 = pack2<FP8>(p0 - f0.x, p1 - f0.y);
        bl1 = pack2<FP8>(p2 - f1.x, p3 - f1.y);
      }
      // V rows 16u + 2t + {0, 1, 8, 9}: the dims of lane group g
      const uint8_t* Vu = Vs + 16 * u * RB;
      if constexpr (RB == 64) {     // FP8, D = 64: 8 bytes (8 dims) of lane group g per row
        uint2 x[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const uint2*>(Vu + voff[i][0]);
#pragma unroll
        for (int e = 0; e < 2; ++e) {            // word e: dims 8g + 4e .. +3 = m-tiles 2e, 2e+1
          const uint32_t w0 = e ? x[0].y : x[0].x, w1 = e ? x[1].y : x[1].x;
          const uint32_t w8 = e ? x[2].y : x[2].x, w9 = e ? x[3].y : x[3].x;
          const uint32_t lo01 = prmt(w0, w1, 0x5140), hi01 = prmt(w0, w1, 0x7362);
          const uint32_t lo89 = prmt(w8, w9, 0x5140), hi89 = prmt(w8, w9, 0x7362);
          const uint32_t A0 = e4m3x2_to_f16x2(lo01 & 0xFFFF), A1 = e4m3x2_to_f16x2(lo01 >> 16);
          const uint32_t A2 = e4m3x2_to_f16x2(lo89 & 0xFFFF), A3 = e4m3x2_to_f16x2(lo89 >> 16);
          const uint32_t B0 = e4m3x2_to_f16x2(hi01 & 0xFFFF), B1 = e4m3x2_to_f16x2(hi01 >> 16);
          const uint32_t B2 = e4m3x2_to_f16x2(hi89 & 0xFFFF), B3 = e4m3x2_to_f16x2(hi89 >> 16);
          mma16816<true>(oacc[2 * e], A0, A1, A2, A3, bh0, bh1);
          mma16816<true>(oacc[2 * e], A0, A1, A2, A3, bl0, bl1);
          mma16816<true>(oacc[2 * e + 1], B0, B1, B2, B3, bh0, bh1);
          mma16816<true>(oacc[2 * e + 1], B0, B1, B2, B3, bl0, bl1);
        }
      } else {
        constexpr int VCH = RB == 256 ? 2 : 1;   // 16-byte chunks of a lane group per row
#pragma unroll
        for (int ci = 0; ci < VCH; ++ci) {
          uint4 x[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const uint4*>(Vu + voff[i][ci]);
          const uint32_t w0[4] = {x[0].x, x[0].y, x[0].z, x[0].w};
          const uint32_t w1[4] = {x[1].x, x[1].y, x[1].z, x[1].w};
          const uint32_t w8[4] = {x[2].x, x[2].y, x[2].z, x[2].w};
          const uint32_t w9[4] = {x[3].x, x[3].y, x[3].z, x[3].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if constexpr (FP8) {     // word e: 4 dims = m-tiles 2e, 2e + 1
              const uint32_t lo01 = prmt(w0[e], w1[e], 0x5140), hi01 = prmt(w0[e], w1[e], 0x7362);
              const uint32_t lo89 = prmt(w8[e], w9[e], 0x5140), hi89 = prmt(w8[e], w9[e], 0x7362);
              const uint32_t A0 = e4m3x2_to_f16x2(lo01 & 0xFFFF),
                             A1 = e4m3x2_to_f16x2(lo01 >> 16);
              const uint32_t A2 = e4m3x2_to_f16x2(lo89 & 0xFFFF),
                             A3 = e4m3x2_to_f16x2(lo89 >> 16);
              const uint32_t B0 = e4m3x2_to_f16x2(hi01 & 0xFFFF),
                             B1 = e4m3x2_to_f16x2(hi01 >> 16);
              const uint32_t B2 = e4m3x2_to_f16x2(hi89 & 0xFFFF),
                             B3 = e4m3x2_to_f16x2(hi89 >> 16);
              mma16816<true>(oacc[2 * e], A0, A1, A2, A3, bh0, bh1);
              mma16816<true>(oacc[2 * e], A0, A1, A2, A3, bl0, bl1);
              mma16816<true>(oacc[2 * e + 1], B0, B1, B2, B3, bh0, bh1);
              mma16816<true>(oacc[2 * e + 1], B0, B1, B2, B3, bl0, bl1);
            } else {                 // word e: 2 dims = m-tile 4 ci + e (rows g, g + 8)
              const int i = 4 * ci + e;
              const uint32_t a0 = prmt(w0[e], w1[e], 0x5410), a1 = prmt(w0[e], w1[e], 0x7632);
              const uint32_t a2 = prmt(w8[e], w9[e], 0x5410), a3 = prmt(w8[e], w9[e], 0x7632);
              mma16816<false>(oacc[i], a0, a1, a2, a3, bh0, bh1);
              mma16816<false>(oacc[i], a0, a1, a2, a3, bl0, bl1);
            }
          }
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
    if (lane == 0 && k + SPW < nt) issue(ring[(k + SPW) % NMR], k + SPW);

    // ---- end of this head inside the range
    if (mt.flags & kLast) {
      float l = l_run;
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      const int hidx = mt.hidx;
      const int kb = hidx / c.Hkv, kh = hidx % c.Hkv;
      if constexpr (CS > 0) {   // the warp's partial, for the CTA's merge
        float* po = mslot + warp * T::SLOT;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * t + e;
          if (h < G) {
#pragma unroll
            for (int i = 0; i < MT; ++i) {
              po[h * D + T::vdim(g, i, 0)] = oacc[i][e] * mt.vhead;
              po[h * D + T::vdim(g, i, 1)] = oacc[i][2 + e] * mt.vhead;
            }
          }
        }
        if (t == 0 && g < G) {
          po[G * D + g] = m_run;
          po[G * D + G + g] = l;
        }
      } else if (page_off[hidx] >= gp0 && page_off[hidx + 1] <= gp0 + nt) {
        // the whole head lies in this warp's range: write the output now
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * t + e;
          const float lh = __shfl_sync(0xffffffffu, l, 4 * (h & 7));
          const float mh = __shfl_sync(0xffffffffu, m_run, 4 * (h & 7));
          if (h < G) {
            const float inv = mh == -INFINITY ? 0.f : mt.vhead / lh;
            const long long ob = ((long long)kb * c.Hq + (long long)kh * G + h) * D;
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
              for (int hi = 0; hi < 2; ++hi) {
                const float o = oacc[i][2 * hi + e] * inv;
                const long long oi = ob + T::vdim(g, i, hi);
                if (oa.f32) static_cast<float*>(oa.out)[oi] = o;
                else static_cast<uint16_t*>(oa.out)[oi] = f32_to_bf16_rn(o);
              }
            if (oa.lse && g == 0)
              oa.lse[(long long)kb * c.Hq + kh * G + h] =
                  mh == -INFINITY ? -INFINITY : (mh + log2f(lh)) * 0.6931471805599453f;
          }
        }
      } else {
        // shared with other warps: this warp's partial goes to the workspace,
        // at v + hidx (unique: a warp's heads are consecutive, and later
        // warps never go back to earlier heads)
        const long long part = v_range + hidx;
        float* po = w.part_o + part * G * D;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * t + e;
          if (h < G) {
#pragma unroll
            for (int i = 0; i < MT; ++i) {
              po[h * D + T::vdim(g, i, 0)] = oacc[i][e] * mt.vhead;
              po[h * D + T::vdim(g, i, 1)] = oacc[i][2 + e] * mt.vhead;
            }
          }
        }
        if (t == 0 && g < G) {
          w.part_ml[(part * G + g) * 2] = m_run;
          w.part_ml[(part * G + g) * 2 + 1] = l;
        }
      }
    }
  }

  if constexpr (CS > 0) {
    // ---- merge: the warps' partials into the CTA's (shared memory), then the
    // CTAs' partials across the cluster; each CTA writes 1/CS of the head's
    // output. o = sum_w 2^(m_w - M) o_w / sum_w 2^(m_w - M) l_w.
    __syncthreads();
    float* cp = mslot + T::NCW * T::SLOT;
    for (int e = tid; e < G * D; e += T::NT) {
      const int h = e / D;
      float M = -INFINITY;
#pragma unroll
      for (int v = 0; v < T::NCW; ++v) M = fmaxf(M, mslot[v * T::SLOT + G * D + h]);
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int v = 0; v < T::NCW; ++v) {
          const float mv = mslot[v * T::SLOT + G * D + h];
          if (mv != -INFINITY) {   // empty partials hold no o values
            const float bw = fast_exp2(mv - M);
            L += mslot[v * T::SLOT + G * D + G + h] * bw;
            O += mslot[v * T::SLOT + e] * bw;
          }
        }
      }
      cp[e] = O;
      if (e % D == 0) {
        cp[G * D + h] = M;
        cp[G * D + G + h] = L;
      }
    }
    __syncthreads();   // converged warps for the aligned cluster barrier
    cluster_sync_all();
    const int kb = hsel / c.Hkv, kh = hsel % c.Hkv;
    const int crank = (int)(blockIdx.x % CS);
    constexpr int PER = G * D / CS;
    for (int e = crank * PER + tid; e < (crank + 1) * PER; e += T::NT) {
      const int h = e / D, d = e % D;
      float M = -INFINITY, L = 0.f, O = 0.f;
#pragma unroll
      for (int j = 0; j < CS; ++j) {
        const float mj = ld_cluster_f32(cp + G * D + h, (uint32_t)j);
        if (mj == -INFINITY) continue;
        const float lj = ld_cluster_f32(cp + G * D + G + h, (uint32_t)j);
        const float oj = ld_cluster_f32(cp + e, (uint32_t)j);
        const float mx = fmaxf(M, mj);
        const float a = fast_exp2(M - mx), bw = fast_exp2(mj - mx);   // a = 0 while M = -inf
        L = L * a + lj * bw;
        O = O * a + oj * bw;
        M = mx;
      }
      const float o = M == -INFINITY ? 0.f : O / L;
      const long long oi = ((long long)kb * c.Hq + (long long)kh * G + h) * D + d;
      if (oa.f32) static_cast<float*>(oa.out)[oi] = o;
      else static_cast<uint16_t*>(oa.out)[oi] = f32_to_bf16_rn(o);
      if (oa.lse && d == 0)
        oa.lse[(long long)kb * c.Hq + kh * G + h] =
            M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
    }
    __syncthreads();
    cluster_sync_all();   // no CTA leaves while another still reads its shared memory
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
// Cluster size for a call of nh heads: the largest of 8, 4, 2 whose nh * CS
// CTAs fit on the SMs at once, if the call has at most half as many heads as
// there are SMs; 0 selects the global plan and the combine kernel, which a
// cache created with an explicit split grid (decode_ctas > 0) always uses.
inline int cluster_size(const fdms_cache* cache, int nh) {
#if FDMS_CLUSTER_DECODE
  if (!cache->cluster_ok || cache->cfg.decode_ctas > 0) return 0;
  for (int cs = 8; cs >= 2; cs /= 2)
    if ((long long)nh * cs <= cache->num_sms) return cs;
#endif
  (void)cache;
  (void)nh;
  return 0;
}

template <class T, int CS>
fdms_status launch_cluster_t(fdms_cache* cache, const DecodeWork& w, OutArgs oa, int layer,
                             int batch, const void* q, cudaStream_t s) {
  const int nh = batch * cache->view.Hkv;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nh * CS));
  cfg.blockDim = dim3(T::NT);
  cfg.dynamicSmemBytes = T::smem_bytes_cluster(nh);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_decode_split<T, CS>, cache->view, w, oa,
                                           layer, batch, static_cast<const uint16_t*>(q), 0,
                                           0.0);
  if (e != cudaSuccess) return FDMS_ERR_CUDA;
  cache->last_append_layer = -1;   // the kernel waits for every append queued before it
  return FDMS_OK;
}

template <class T>
fdms_status launch_split_t(fdms_cache* cache, const DecodeWork& w, OutArgs oa, int layer,
                           int batch, const void* q, cudaStream_t s) {
  const int nh = batch * cache->view.Hkv;
  switch (cluster_size(cache, nh)) {
    case 8: return launch_cluster_t<T, 8>(cache, w, oa, layer, batch, q, s);
    case 4: return launch_cluster_t<T, 4>(cache, w, oa, layer, batch, q, s);
    case 2: return launch_cluster_t<T, 2>(cache, w, oa, layer, batch, q, s);
    default: break;
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
                                     1.0 / (double)n_ranges);
  if (e != cudaSuccess) return FDMS_ERR_CUDA;
  cache->last_append_layer = -1;   // the split waits for every append queued before it
  cfg.gridDim = dim3((unsigned)(nh * Combine<T::D, T::G>::CPH));
  cfg.blockDim = dim3(Combine<T::D, T::G>::NT);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, k_decode_combine<T::D, T::G, T::TR>, cache->view, w, layer, batch,
                         oa, n_ranges, 1.0 / (double)n_ranges);
  return e == cudaSuccess ? FDMS_OK : FDMS_ERR_CUDA;
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
  // per-head cluster mode: usable when every cluster size fits
  const size_t csmem = T::smem_bytes_cluster(nh);
  cache->cluster_ok =
      csmem <= 227 * 1024 &&
      cudaFuncSetAttribute(k_decode_split<T, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)csmem) == cudaSuccess &&
      cudaFuncSetAttribute(k_decode_split<T, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)csmem) == cudaSuccess &&
      cudaFuncSetAttribute(k_decode_split<T, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)csmem) == cudaSuccess;
  cudaGetLastError();   // a refused attribute only turns the cluster mode off
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
  w.part_o = static_cast<float*>(take((size_t)w.max_parts * c.G * c.D * sizeof(float)));
  w.part_ml = static_cast<float*>(take((size_t)w.max_parts * c.G * 2 * sizeof(float)));
  if (!w.part_o || !w.part_ml) return FDMS_ERR_CUDA;
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
// A fixed scratch array for fdms_decode_attn_noalloc: the split plan and the
// split partials. Host code only learns its device address through
// cudaGetSymbolAddress (the host-side name is a stand-in, not a device
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

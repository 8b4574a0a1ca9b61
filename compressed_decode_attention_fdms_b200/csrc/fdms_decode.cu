// Decode attention over the compact store: split kernel + combine kernel.
//
// FastDMS decodes over the survivors of per-head eviction only, reading 5-8x
// less KV than a dense cache ("FastDMS: 6.4X KV-cache compression running
// faster than vLLM BF16/FP8", aiwitness.kr/community/1t3vlrx, paragraph on
// decode speed and memory at 8K context). For query head g of kv head h:
//     o_g = sum_{j in S_h} softmax_j(scale * q_g . k_j) v_j,
// S_h = the head's compact store plus its visible ring slots.
//
// Split kernel (memory bound: every byte of a visible K and V row is read once):
//   - Work is balanced over the GPU by slots, not by heads. The slot lists of
//     all heads of the call are laid end to end (units = store slots + ring
//     slots) and cut into equal ranges, one per consumer warp of the grid; a
//     warp therefore reads the same number of bytes whatever the mix of head
//     lengths, and emits one partial (m, l, o) per head its range touches.
//   - A producer warp walks each consumer warp's pages (64 rows of a store
//     block, or 64 ring slots; 32 rows when a row is 256 bytes) and stages a
//     page's K rows, V rows and the head's q into shared memory with 1-D bulk
//     copies (cp.async.bulk, completion on an mbarrier). Rows keep their page
//     row in shared memory, so the chunk permutation they are stored with
//     makes the fragment loads below free of bank conflicts. Every consumer
//     warp owns two stages (double buffering) and never waits for another.
//   - A consumer warp computes the G x 64 scores of a page on the tensor cores
//     (mma.sync m16n8k16, fp32 accumulate; the G query heads sharing the kv
//     head are rows 0..G-1 of the 16-row tile), an online softmax in fp32 in
//     the log2 domain, and p.v on the tensor cores again. p is split into a
//     16-bit head and a 16-bit remainder so its rounding stays below 2^-16.
//     BF16 pages feed the bf16 MMA directly. FP8 pages are converted exactly
//     to f16 (cvt e4m3x2 -> f16x2) and q is brought into f16 range by a power
//     of two that the score scale undoes; the page's K scale multiplies the
//     scores and its V scale the probabilities, never the elements.
// Combine kernel: per (seq, kv head) the partials of the warps that covered it
// are merged: o = sum_w 2^(m_w - M) o_w / sum_w 2^(m_w - M) l_w.
#include <cfloat>
#include <cstdio>
#include <mutex>

#include "fdms_internal.cuh"

namespace fdms {
namespace {

constexpr int kMinUnitsPerRange = 64;  // a consumer warp gets at least one page of work
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

enum : int { kFirst = 1, kLast = 2, kRing = 4, kPending = 8 };

struct TileMeta {
  int hidx;      // head of the call (b * Hkv + h)
  int row0;      // rows [row0, row1) of the page frame hold this tile's slots
  int row1;
  int flags;
  int p0;        // ring tiles: position of row row0
  int thresh;    // ring tiles: positions below n - W need their keep bit
  int R;         // ring capacity (slot = p % R)
  float ks;      // K scale of the page
  float vrel;    // V scale of the page / the head's V scale
  float vhead;   // the head's V scale (1 for BF16)
  long long keep_base;   // ring tiles: index of the head's ring_keep
};

template <int D_, bool FP8_, int G_>
struct Dec {
  static constexpr int D = D_, G = G_;
  static constexpr bool FP8 = FP8_;
  static constexpr int ELT = FP8 ? 1 : 2;
  static constexpr int RB = D * ELT;           // bytes per row
  static constexpr int TR = RB <= 128 ? 64 : 32;   // rows per tile (a page or half a page)
  static constexpr int NCW = 4;                // consumer warps
  static constexpr int NC = NCW * 32;
  static constexpr int NT = NC + 32;           // + one producer warp
  static constexpr int SPW = 2;                // stages per consumer warp
  static constexpr int NSTAGE = NCW * SPW;
  static constexpr int KV_BYTES = TR * RB;
  static constexpr int Q_BYTES = G * D * 2;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES + ((Q_BYTES + 127) / 128) * 128;
  static constexpr int NJ = TR / 8;            // score n-tiles (8 keys each)
  static constexpr int NU = TR / 16;           // p.v k-steps (16 keys each)
  static constexpr int KS = D / 16;            // q.k k-steps (16 dims each)
  static constexpr int ND = D / 8;             // p.v n-tiles (8 dims each)
  static constexpr int EC = 16 / ELT;          // elements per 16-byte chunk
  static constexpr int KCPT = (RB / 16) / 4;   // K chunks per thread (1, 2 or 4)
  static_assert(NSTAGE <= 32, "one producer lane per stage");

  static constexpr int OFF_META = NSTAGE * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_META + NSTAGE * (int)sizeof(TileMeta);
  static constexpr int OFF_HEADS = OFF_BAR + 2 * NSTAGE * 8;
  static size_t smem_bytes(int nh) {
    // head_off (i64), page_off (i32), len, n, r (i32), head scales (2 x f32)
    return 128 + OFF_HEADS + (size_t)(nh + 1) * 8 + (size_t)(nh + 1) * 4 +
           (size_t)nh * 4 * 3 + (size_t)nh * 8 + 64;
  }

  // unpermuted 16-byte K chunk i (0 .. KCPT-1) of lane column t
  __device__ static int kchunk(int t, int i) { return RB == 256 ? t + 4 * i : KCPT * t + i; }
  // element (dim) of the row behind k-step s, slot e (0..3) of lane column t:
  // e = 0, 1 are the fragment's k = 2t, 2t+1; e = 2, 3 are k = 2t+8, 2t+9
  __device__ static int kdim(int t, int s, int e) {
    const int se = 4 * s + e;
    return kchunk(t, se / EC) * EC + se % EC;
  }
  // dim held by p.v n-tile d in the B columns of lane group g
  __device__ static int vdim(int g, int d) {
    if (RB == 256) return d < 8 ? 8 * g + d : 64 + 8 * g + (d - 8);
    return ND * g + d;   // RB 128: 8 (bf16) or 16 (fp8) dims per lane group; RB 64: 8
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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

template <class T>
__device__ __forceinline__ int upper_bound(const T* a, int n, T x) {
  int lo = 0, hi = n;   // first index with a[i] > x
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] <= x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------------- MMA helpers
template <bool F16>
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
  // A rows 8..15 are padding (zero): a1 = a3 = 0
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
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

template <class T>
__global__ void __launch_bounds__(T::NT, 1)
k_decode_split(CacheView c, DecodeWork w, int layer, int batch, const uint16_t* __restrict__ q,
               int n_launch_ranges) {
  constexpr int D = T::D, G = T::G, RB = T::RB, TR = T::TR, NSTAGE = T::NSTAGE,
                NCW = T::NCW, SPW = T::SPW, NJ = T::NJ, NU = T::NU, KS = T::KS, ND = T::ND;
  constexpr bool FP8 = T::FP8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  TileMeta* meta = reinterpret_cast<TileMeta*>(smem + T::OFF_META);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  uint64_t* empty = full + NSTAGE;
  const int NH = batch * c.Hkv;
  long long* head_off = reinterpret_cast<long long*>(smem + T::OFF_HEADS);   // [NH + 1]
  int* page_off = reinterpret_cast<int*>(head_off + NH + 1);                 // [NH + 1]
  int* s_len = page_off + NH + 1;
  int* s_n = s_len + NH;
  int* s_r = s_n + NH;
  float* s_hscale = reinterpret_cast<float*>(s_r + NH);                      // [NH][2]

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long hi0 = (long long)layer * c.Bmax * c.Hkv;   // first head of this layer

  // stale rows of a stage are multiplied by p = 0: start from zeros, not from
  // whatever bits shared memory held
  for (int i = tid; i < NSTAGE * T::STAGE_BYTES / 16; i += T::NT)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);

  // ---- 1. units and pages of every head of the call; exclusive prefix
  {
    const int per = (NH + T::NT - 1) / T::NT;
    const int h0 = tid * per, h1 = min(NH, h0 + per);
    long long su = 0;
    int sp = 0;
    auto pages = [](int len, int live, int r) {
      return (len + TR - 1) / TR + (live > 0 ? (live + (r % TR) + TR - 1) / TR : 0);
    };
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
  const long long total = head_off[NH];
  const long long want = (total + kMinUnitsPerRange - 1) / kMinUnitsPerRange;
  const int n_eff = (int)(want < n_launch_ranges ? (want > 0 ? want : 1) : n_launch_ranges);
  if (blockIdx.x == 0) {
    for (int h = tid; h <= NH; h += T::NT) w.head_off[h] = head_off[h];
    if (tid == 0) {
      *w.n_eff = n_eff;
      c.ctr->slots_decoded += (unsigned long long)total;   // one CTA, launches are ordered
      c.ctr->decode_calls += 1ull;
    }
  }
  if ((int)blockIdx.x * NCW >= n_eff || total == 0) return;

  // page (in the call's page numbering) holding global unit x
  auto gpage = [&](long long x) -> int {
    const int h = upper_bound(head_off, NH + 1, x) - 1;
    const long long u = x - head_off[h];
    const int len = s_len[h];
    const int lp = u < len ? (int)(u / TR)
                           : (len + TR - 1) / TR + (int)((u - len + s_r[h] % TR) / TR);
    return page_off[h] + lp;
  };
  // unit range of consumer warp cw of this CTA, and its first page / page count
  auto range_of = [&](int cw, long long& gs, long long& ge, int& gp0, int& nt) {
    const long long v = (long long)blockIdx.x * NCW + cw;
    nt = 0;
    gs = ge = 0;
    gp0 = 0;
    if (v >= n_eff) return;
    gs = v * total / n_eff;
    ge = (v + 1) * total / n_eff;
    if (gs >= ge) return;
    gp0 = gpage(gs);
    nt = gpage(ge - 1) - gp0 + 1;
  };

  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ================= producer: lane l owns stage l, i.e. consumer warp l / SPW
    // and that warp's tiles l % SPW, l % SPW + SPW, ...
    if (lane < NSTAGE) {
      const int cw = lane / SPW;
      long long gs, ge;
      int gp0, nt;
      range_of(cw, gs, ge, gp0, nt);
      for (int k = lane % SPW; k < nt; k += SPW) {
        const int gp = gp0 + k;
        const int hidx = upper_bound(page_off, NH + 1, gp) - 1;
        const int lp = gp - page_off[hidx];
        const int len = s_len[hidx], n = s_n[hidx], r = s_r[hidx];
        const int sp = (len + TR - 1) / TR;
        const long long hoff = head_off[hidx];
        const long long lo = gs > hoff ? gs - hoff : 0;   // head units of this range
        const long long hi_u = ge - hoff;
        const long long hi = hi0 + hidx;
        TileMeta mt;
        mt.hidx = hidx;
        mt.flags = (k == 0 || lp == 0 ? kFirst : 0) |
                   (k == nt - 1 || gp + 1 == page_off[hidx + 1] ? kLast : 0);
        mt.vhead = s_hscale[2 * hidx + 1];
        mt.p0 = mt.thresh = mt.R = 0;
        mt.keep_base = 0;
        const uint8_t *ksrc, *vsrc;
        if (lp < sp) {   // store page lp: block lp * TR / 64, rows from (lp * TR) % 64
          const long long u0 = max((long long)lp * TR, lo);
          const long long u1 = min((long long)min((lp + 1) * TR, len), hi_u);
          const int j = lp * TR / kBlockSlots;
          const int rb = (lp * TR) % kBlockSlots;          // block row of frame row 0
          mt.row0 = (int)(u0 - (long long)lp * TR);
          mt.row1 = (int)(u1 - (long long)lp * TR);
          const long long blk = c.block_table[hi * c.max_blocks + j];
          if (FP8) {
            mt.ks = c.bt_scale[(hi * c.max_blocks + j) * 2];
            mt.vrel = c.bt_scale[(hi * c.max_blocks + j) * 2 + 1] / mt.vhead;
          } else {
            mt.ks = mt.vrel = 1.0f;
          }
          ksrc = block_k(c, blk) + (long long)(rb + mt.row0) * RB;
          vsrc = block_v(c, blk) + (long long)(rb + mt.row0) * RB;
        } else {         // ring page: live units [TR*rp - off, TR*(rp+1) - off)
          const int rp = lp - sp, off = r % TR, live = n - r;
          const long long a = max((long long)len + max(TR * rp - off, 0), lo);
          const long long b = min((long long)len + min(TR * (rp + 1) - off, live), hi_u);
          const int p0 = r + (int)(a - len);
          const int slot0 = p0 % c.R;
          mt.row0 = slot0 % TR;
          mt.row1 = mt.row0 + (int)(b - a);
          mt.p0 = p0;
          mt.thresh = n - c.W;
          mt.R = c.R;
          mt.keep_base = hi * c.Rpad;
          mt.flags |= kRing | (p0 < mt.thresh ? kPending : 0);
          mt.ks = s_hscale[2 * hidx];
          mt.vrel = 1.0f;
          ksrc = ring_k(c, hi) + (long long)slot0 * RB;
          vsrc = ring_v(c, hi) + (long long)slot0 * RB;
        }
        const int s = lane;
        const int use = k / SPW;
        if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1)) {
          latch_error(c.ctr, FDMS_ERR_DEVICE);
          break;
        }
        meta[s] = mt;
        uint8_t* kdst = smem + s * T::STAGE_BYTES;
        uint8_t* vdst = kdst + T::KV_BYTES;
        const uint32_t rows = (uint32_t)(mt.row1 - mt.row0);
        mbar_arrive_expect_tx(&full[s], 2u * rows * RB + (uint32_t)T::Q_BYTES);
        bulk_g2s(kdst + mt.row0 * RB, ksrc, rows * RB, &full[s]);
        bulk_g2s(vdst + mt.row0 * RB, vsrc, rows * RB, &full[s]);
        const int b = hidx / c.Hkv, h = hidx % c.Hkv;
        bulk_g2s(vdst + T::KV_BYTES, q + ((long long)b * c.Hq + (long long)h * G) * D, T::Q_BYTES,
                 &full[s]);
      }
    }
    return;
  }

  // ================= consumer warp `warp`
  const int g = lane >> 2, t = lane & 3;
  long long gs, ge;
  int gp0, nt;
  range_of(warp, gs, ge, gp0, nt);
  const long long range_id = (long long)blockIdx.x * NCW + warp;
  const float qscale = c.softmax_scale * kLog2e;

  uint32_t qa[KS][2];          // q A-fragments (row g, k-steps)
  float qmul = 0.f;            // score multiplier of row g (scale, log2 e, q's power of two)
  int cur_hidx = -1;
  float m_run = -INFINITY, l_run = 0.f;
  float oacc[ND][4];
#pragma unroll
  for (int d = 0; d < ND; ++d) oacc[d][0] = oacc[d][1] = oacc[d][2] = oacc[d][3] = 0.f;

  for (int k = 0; k < nt; ++k) {
    const int s = warp * SPW + (k % SPW);
    const bool ok = mbar_wait(&full[s], (k / SPW) & 1);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
      break;
    }
    const TileMeta mt = meta[s];
    const uint8_t* Ks = smem + s * T::STAGE_BYTES;
    const uint8_t* Vs = Ks + T::KV_BYTES;
    const uint16_t* Qs = reinterpret_cast<const uint16_t*>(Vs + T::KV_BYTES);
    const int row0 = mt.row0, row1 = mt.row1;

    // ---- q fragments of the head (only when the head changes)
    if (mt.hidx != cur_hidx) {
      cur_hidx = mt.hidx;
      if constexpr (FP8) {
        // f16 q scaled by 2^a so that max |q| of the row is in [2^14, 2^15)
        float amax = 0.f;
        if (g < G) {
#pragma unroll
          for (int s2 = 0; s2 < KS; ++s2)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              amax = fmaxf(amax,
                           fabsf(__uint_as_float((uint32_t)Qs[g * D + T::kdim(t, s2, e)] << 16)));
        }
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
          float v4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            v4[e] = g < G ? __uint_as_float((uint32_t)Qs[g * D + T::kdim(t, s2, e)] << 16) * up
                          : 0.f;
          qa[s2][0] = pack2<true>(v4[0], v4[1]);
          qa[s2][1] = pack2<true>(v4[2], v4[3]);
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
      for (int d = 0; d < ND; ++d) oacc[d][0] = oacc[d][1] = oacc[d][2] = oacc[d][3] = 0.f;
    }

    // ---- scores of rows 8j + (0..7): S[head g][keys 8j + 2t, 8j + 2t + 1]
    float sc[NJ][2];
    const float mul = qmul * mt.ks;
    const bool pend = (mt.flags & kPending) != 0;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      sc[j][0] = sc[j][1] = -INFINITY;
      if (8 * j + 8 <= row0 || 8 * j >= row1) continue;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const int r = 8 * j + g;   // key row this lane loads for the B fragment
      uint32_t kw[T::KCPT][4];
#pragma unroll
      for (int i = 0; i < T::KCPT; ++i) {
        const uint4 x = *reinterpret_cast<const uint4*>(
            Ks + r * RB + 16 * swz_chunk(RB, false, r, T::kchunk(t, i)));
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
        mma16816<FP8>(acc, qa[s2][0], qa[s2][1], b0, b1);
      }
      const int ra = 8 * j + 2 * t;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = ra + e;
        bool vis = row >= row0 && row < row1;
        if (vis && pend) {
          const int p = mt.p0 + (row - row0);
          if (p < mt.thresh) vis = c.ring_keep[mt.keep_base + p % mt.R] != 0;
        }
        sc[j][e] = vis ? acc[e] * mul : -INFINITY;
      }
    }

    // ---- online softmax for row g (the 4 lanes of a quad share it)
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < NJ; ++j) mx = fmaxf(mx, fmaxf(sc[j][0], sc[j][1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mn = fmaxf(m_run, mx);
    float alpha = 1.f;
    float pr[NJ][2];
    if (mn == -INFINITY) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) pr[j][0] = pr[j][1] = 0.f;
    } else {
      alpha = fast_exp2(m_run - mn);
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        pr[j][0] = fast_exp2(sc[j][0] - mn);
        pr[j][1] = fast_exp2(sc[j][1] - mn);
        ls += pr[j][0] + pr[j][1];
      }
      l_run = l_run * alpha + ls;
      m_run = mn;
    }
#pragma unroll
    for (int d = 0; d < ND; ++d) {
      oacc[d][0] *= alpha;
      oacc[d][1] *= alpha;
    }

    // ---- o += p v, keys 16u .. 16u + 15 per k-step
#pragma unroll
    for (int u = 0; u < NU; ++u) {
      if (16 * u + 16 <= row0 || 16 * u >= row1) continue;
      const float v0 = pr[2 * u][0] * mt.vrel, v1 = pr[2 * u][1] * mt.vrel;
      const float v2 = pr[2 * u + 1][0] * mt.vrel, v3 = pr[2 * u + 1][1] * mt.vrel;
      const uint32_t ah0 = pack2<FP8>(v0, v1), ah2 = pack2<FP8>(v2, v3);
      const float2 f0 = unpack2<FP8>(ah0), f2 = unpack2<FP8>(ah2);
      const uint32_t al0 = pack2<FP8>(v0 - f0.x, v1 - f0.y);
      const uint32_t al2 = pack2<FP8>(v2 - f2.x, v3 - f2.y);
      // V rows 16u + 2t + {0, 1, 8, 9}: the dims of lane group g
      const int rr[4] = {16 * u + 2 * t, 16 * u + 2 * t + 1, 16 * u + 2 * t + 8,
                         16 * u + 2 * t + 9};
      if constexpr (RB == 64) {     // FP8, D = 64: 8 bytes (8 dims) per row
        uint2 x[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          x[i] = *reinterpret_cast<const uint2*>(Vs + rr[i] * RB + 8 * g);
#pragma unroll
        for (int e = 0; e < 2; ++e) {            // words: dims 4e .. 4e + 3
          const uint32_t a0w = e ? x[0].y : x[0].x, a1w = e ? x[1].y : x[1].x;
          const uint32_t a8w = e ? x[2].y : x[2].x, a9w = e ? x[3].y : x[3].x;
          const uint32_t lo01 = prmt(a0w, a1w, 0x5140), hi01 = prmt(a0w, a1w, 0x7362);
          const uint32_t lo89 = prmt(a8w, a9w, 0x5140), hi89 = prmt(a8w, a9w, 0x7362);
          const uint32_t b0s[4] = {e4m3x2_to_f16x2(lo01 & 0xFFFF), e4m3x2_to_f16x2(lo01 >> 16),
                                   e4m3x2_to_f16x2(hi01 & 0xFFFF), e4m3x2_to_f16x2(hi01 >> 16)};
          const uint32_t b1s[4] = {e4m3x2_to_f16x2(lo89 & 0xFFFF), e4m3x2_to_f16x2(lo89 >> 16),
                                   e4m3x2_to_f16x2(hi89 & 0xFFFF), e4m3x2_to_f16x2(hi89 >> 16)};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            mma16816<true>(oacc[4 * e + q4], ah0, ah2, b0s[q4], b1s[q4]);
            mma16816<true>(oacc[4 * e + q4], al0, al2, b0s[q4], b1s[q4]);
          }
        }
      } else {
        constexpr int VCH = RB == 256 ? 2 : 1;   // 16-byte chunks of a lane group per row
#pragma unroll
        for (int ci = 0; ci < VCH; ++ci) {
          const int chunk = RB == 256 ? g + 8 * ci : g;
          uint4 x[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            x[i] = *reinterpret_cast<const uint4*>(Vs + rr[i] * RB +
                                                  16 * swz_chunk(RB, true, rr[i], chunk));
          const uint32_t w0[4] = {x[0].x, x[0].y, x[0].z, x[0].w};
          const uint32_t w1[4] = {x[1].x, x[1].y, x[1].z, x[1].w};
          const uint32_t w8[4] = {x[2].x, x[2].y, x[2].z, x[2].w};
          const uint32_t w9[4] = {x[3].x, x[3].y, x[3].z, x[3].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if constexpr (FP8) {                 // 4 dims per word: n-tiles 4e .. 4e + 3
              const uint32_t lo01 = prmt(w0[e], w1[e], 0x5140), hi01 = prmt(w0[e], w1[e], 0x7362);
              const uint32_t lo89 = prmt(w8[e], w9[e], 0x5140), hi89 = prmt(w8[e], w9[e], 0x7362);
              const uint32_t b0s[4] = {e4m3x2_to_f16x2(lo01 & 0xFFFF), e4m3x2_to_f16x2(lo01 >> 16),
                                       e4m3x2_to_f16x2(hi01 & 0xFFFF), e4m3x2_to_f16x2(hi01 >> 16)};
              const uint32_t b1s[4] = {e4m3x2_to_f16x2(lo89 & 0xFFFF), e4m3x2_to_f16x2(lo89 >> 16),
                                       e4m3x2_to_f16x2(hi89 & 0xFFFF), e4m3x2_to_f16x2(hi89 >> 16)};
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                mma16816<true>(oacc[4 * e + q4], ah0, ah2, b0s[q4], b1s[q4]);
                mma16816<true>(oacc[4 * e + q4], al0, al2, b0s[q4], b1s[q4]);
              }
            } else {                              // 2 dims per word: n-tiles 2e, 2e + 1
              const int d0 = 8 * ci + 2 * e;
              const uint32_t b0a = prmt(w0[e], w1[e], 0x5410), b1a = prmt(w8[e], w9[e], 0x5410);
              const uint32_t b0b = prmt(w0[e], w1[e], 0x7632), b1b = prmt(w8[e], w9[e], 0x7632);
              mma16816<false>(oacc[d0], ah0, ah2, b0a, b1a);
              mma16816<false>(oacc[d0], al0, al2, b0a, b1a);
              mma16816<false>(oacc[d0 + 1], ah0, ah2, b0b, b1b);
              mma16816<false>(oacc[d0 + 1], al0, al2, b0b, b1b);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    // ---- end of this head inside the range: write the partial
    if (mt.flags & kLast) {
      float l = l_run;
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      const long long part = range_id + mt.hidx;
      if (g < G) {
        float* po = w.part_o + (part * G + g) * D;
#pragma unroll
        for (int d = 0; d < ND; ++d) {
          po[T::vdim(2 * t, d)] = oacc[d][0] * mt.vhead;
          po[T::vdim(2 * t + 1, d)] = oacc[d][1] * mt.vhead;
        }
        if (t == 0) {
          w.part_ml[(part * G + g) * 2] = m_run;
          w.part_ml[(part * G + g) * 2 + 1] = l;
        }
      }
    }
  }
}

// range of unit x under the split: the largest v with floor(v * T / N) <= x.
__device__ __forceinline__ int range_of_unit(long long x, long long total, int n) {
  return (int)(((x + 1) * n - 1) / total);
}

template <int D, int G, bool F32>
__global__ void __launch_bounds__(G * D)
k_decode_combine(DecodeWork w, int Hkv, int Hq, int batch, void* out, float* lse) {
  const int hidx = blockIdx.x;
  const int g = threadIdx.x / D, d = threadIdx.x % D;
  const int b = hidx / Hkv, h = hidx % Hkv;
  const int qh = h * G + g;
  const long long s = w.head_off[hidx], e = w.head_off[hidx + 1];
  const long long total = w.head_off[batch * Hkv];
  const int n = *w.n_eff;
  float o = 0.f, M = -INFINITY, L = 0.f;
  if (e > s) {
    const int c0 = range_of_unit(s, total, n), c1 = range_of_unit(e - 1, total, n);
    for (int cc = c0; cc <= c1; ++cc) {
      const long long part = (long long)cc + hidx;
      M = fmaxf(M, w.part_ml[(part * G + g) * 2]);
    }
    if (M != -INFINITY) {
      for (int cc = c0; cc <= c1; ++cc) {
        const long long part = (long long)cc + hidx;
        const float m = w.part_ml[(part * G + g) * 2];
        if (m == -INFINITY) continue;
        const float sc = exp2f(m - M);
        L += w.part_ml[(part * G + g) * 2 + 1] * sc;
        o += w.part_o[(part * G + g) * D + d] * sc;
      }
      o = o / L;
    }
  }
  const long long oi = ((long long)b * Hq + qh) * D + d;
  if constexpr (F32) {
    static_cast<float*>(out)[oi] = o;
    if (lse && d == 0)
      lse[(long long)b * Hq + qh] =
          (M == -INFINITY) ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
  } else {
    static_cast<uint16_t*>(out)[oi] = f32_to_bf16_rn(o);
  }
}

// ------------------------------------------------------------------ dispatch
template <class T>
fdms_status launch_split_t(fdms_cache* cache, int layer, int batch, const void* q,
                           cudaStream_t s) {
  const int nh = batch * cache->view.Hkv;
  const size_t smem = T::smem_bytes(nh);
  k_decode_split<T><<<cache->decode_ctas, T::NT, smem, s>>>(
      cache->view, cache->work, layer, batch, static_cast<const uint16_t*>(q),
      cache->decode_ctas * T::NCW);
  return cudaGetLastError() == cudaSuccess ? FDMS_OK : FDMS_ERR_CUDA;
}

template <class T>
fdms_status setup_t(fdms_cache* cache) {
  const int nh = cache->view.Bmax * cache->view.Hkv;
  const size_t smem = T::smem_bytes(nh);
  if (smem > 227 * 1024) return FDMS_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(k_decode_split<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return FDMS_ERR_UNSUPPORTED;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode_split<T>, T::NT, smem) !=
          cudaSuccess || per_sm < 1)
    return FDMS_ERR_UNSUPPORTED;
  cache->ctas_per_sm = per_sm;
  cache->ranges_per_cta = T::NCW;
  return FDMS_OK;
}

template <int D, int G, bool F32>
void launch_combine_t(fdms_cache* cache, int batch, void* out, float* lse, cudaStream_t s) {
  const CacheView& c = cache->view;
  k_decode_combine<D, G, F32><<<batch * c.Hkv, G * D, 0, s>>>(cache->work, c.Hkv, c.Hq, batch,
                                                              out, lse);
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
  w.max_parts = ctas * cache->ranges_per_cta + c.Bmax * c.Hkv;
  void* p = nullptr;
  auto take = [&](size_t bytes) -> void* {
    if (cudaMalloc(&p, bytes) != cudaSuccess) return nullptr;
    cache->allocs[cache->nallocs++] = p;
    cache->bytes_reserved += bytes;
    return p;
  };
  w.part_o = static_cast<float*>(take((size_t)w.max_parts * c.G * c.D * sizeof(float)));
  w.part_ml = static_cast<float*>(take((size_t)w.max_parts * c.G * 2 * sizeof(float)));
  w.head_off = static_cast<long long*>(take((size_t)(c.Bmax * c.Hkv + 1) * sizeof(long long)));
  w.n_eff = static_cast<int*>(take(sizeof(int)));
  if (!w.part_o || !w.part_ml || !w.head_off || !w.n_eff) return FDMS_ERR_CUDA;
  return FDMS_OK;
}

fdms_status fdms_launch_decode(fdms_cache* cache, int layer, int batch, const void* q, void* out,
                               int out_f32, float* lse, cudaStream_t s) {
  const CacheView& c = cache->view;
  fdms_status st = by_config(c, [&](auto t) {
    return launch_split_t<decltype(t)>(cache, layer, batch, q, s);
  });
  if (st != FDMS_OK) return st;
  auto comb = [&](auto t) -> fdms_status {
    using T = decltype(t);
    if (out_f32)
      launch_combine_t<T::D, T::G, true>(cache, batch, out, lse, s);
    else
      launch_combine_t<T::D, T::G, false>(cache, batch, out, nullptr, s);
    return cudaGetLastError() == cudaSuccess ? FDMS_OK : FDMS_ERR_CUDA;
  };
  return by_config(c, comb);
}

// ------------------------------------------------- decode without allocation
// A fixed scratch array for fdms_decode_attn_noalloc: the split partials and the
// plan that the combine kernel reads. Host code only learns its device address
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

template <class T>
fdms_status launch_noalloc_t(fdms_cache* cache, const DecodeWork& w, int layer, int batch,
                             const void* q, void* out, cudaStream_t s) {
  const CacheView& c = cache->view;
  const size_t smem = T::smem_bytes(batch * c.Hkv);
  k_decode_split<T><<<cache->decode_ctas, T::NT, smem, s>>>(
      c, w, layer, batch, static_cast<const uint16_t*>(q), cache->decode_ctas * T::NCW);
  if (cudaGetLastError() != cudaSuccess) return FDMS_ERR_CUDA;
  k_decode_combine<T::D, T::G, false><<<batch * c.Hkv, T::G * T::D, 0, s>>>(w, c.Hkv, c.Hq,
                                                                           batch, out, nullptr);
  return cudaGetLastError() == cudaSuccess ? FDMS_OK : FDMS_ERR_CUDA;
}

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
  // layout of the scratch for this call
  const long long parts = (long long)cache->decode_ctas * cache->ranges_per_cta +
                          (long long)batch * c.Hkv;
  const size_t o_bytes = align256((size_t)parts * c.G * c.D * sizeof(float));
  const size_t ml_bytes = align256((size_t)parts * c.G * 2 * sizeof(float));
  const size_t off_bytes = align256((size_t)(batch * c.Hkv + 1) * sizeof(long long));
  const size_t need = o_bytes + ml_bytes + off_bytes + 256;
  if (need > FDMS_STATIC_SCRATCH_BYTES) return FDMS_ERR_INVALID_ARG;

  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return FDMS_ERR_CUDA;
  if (prev != cache->device && cudaSetDevice(cache->device) != cudaSuccess) return FDMS_ERR_CUDA;
  void* base = nullptr;
  fdms_status st = FDMS_OK;
  if (scratch_address(cache->device, &base) != cudaSuccess) {
    st = FDMS_ERR_CUDA;
  } else {
    unsigned char* b = static_cast<unsigned char*>(base);
    DecodeWork w;
    w.part_o = reinterpret_cast<float*>(b);
    w.part_ml = reinterpret_cast<float*>(b + o_bytes);
    w.head_off = reinterpret_cast<long long*>(b + o_bytes + ml_bytes);
    w.n_eff = reinterpret_cast<int*>(b + o_bytes + ml_bytes + off_bytes);
    w.max_parts = (int)parts;
    w.max_ctas = cache->decode_ctas;
    st = by_config(c, [&](auto t) {
      return launch_noalloc_t<decltype(t)>(cache, w, layer, batch, q_dev, out_dev,
                                           static_cast<cudaStream_t>(stream));
    });
  }
  if (prev != cache->device) cudaSetDevice(prev);
  return st;
}

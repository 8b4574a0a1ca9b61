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
//   - Work is balanced over the whole GPU by slots, not by heads: the visible
//     slot lists of all heads of the call are laid end to end (units = store
//     slots + ring slots) and CTA c takes units [c*T/N, (c+1)*T/N). A CTA
//     therefore reads the same number of bytes whatever the mix of lengths;
//     it emits one partial (m, l, o) per head it touches.
//   - A producer warp walks the CTA's 64-slot pages (a store block, or 64 ring
//     slots) and stages each page's K rows and V rows into shared memory with
//     1-D bulk copies (cp.async.bulk, completion on an mbarrier), NSTAGE pages
//     ahead. Each lane of the producer owns one stage, so the block-table load
//     for the next page overlaps the wait for its stage to drain.
//   - Four consumer warps compute the G x 64 scores (fp32, packed f32x2 FMA),
//     an online softmax in the log2 domain, and accumulate p * v, all in fp32.
//     FP8 codes are converted exactly; the block's scales multiply the scores
//     and the probabilities, never the elements.
// Combine kernel: per (seq, kv head) the partials of the CTAs that covered it
// are merged: o = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
#include <cfloat>
#include <cstdio>

#include "fdms_internal.cuh"

namespace fdms {
namespace {

constexpr int kTile = 64;              // rows per page (= pool block)
constexpr int kMinUnitsPerCta = 64;    // a CTA gets at least one page of work
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

enum : int { kFirst = 1, kLast = 2, kRing = 4, kPending = 8 };

struct TileMeta {
  int hidx;      // head of the call (b * Hkv + h)
  int nrows;     // rows staged (<= 64)
  int flags;
  int p0;        // ring tiles: position of row 0
  int thresh;    // ring tiles: positions below n - W need their keep bit
  int R;         // ring capacity (slot = p % R)
  float ks, vs;  // K / V scale of the page
  long long keep_base;   // ring tiles: index of the head's ring_keep
};

template <int D_, bool FP8_, int G_>
struct Dec {
  static constexpr int D = D_, G = G_;
  static constexpr bool FP8 = FP8_;
  static constexpr int ELT = FP8 ? 1 : 2;
  static constexpr int RB = D * ELT;          // bytes per row
  static constexpr int CPR = RB / 16;         // 16-byte chunks per row
  static constexpr int EPC = 16 / ELT;        // elements per chunk
  static constexpr int NCW = 4;               // consumer warps
  static constexpr int NC = NCW * 32;
  static constexpr int NT = NC + 32;          // + one producer warp
  static constexpr int RPP = NC / CPR;        // rows per consumer pass
  static constexpr int NSTAGE = RB <= 128 ? 4 : 3;
  static constexpr int KV_BYTES = kTile * RB;
  static constexpr int Q_BYTES = G * D * 2;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES + ((Q_BYTES + 127) / 128) * 128;
  static_assert(NSTAGE <= 32, "one producer lane per stage");
  static_assert(CPR <= 32 && 32 % CPR == 0, "a row's chunks stay inside one warp");

  // fixed part of shared memory (the per-head arrays follow)
  static constexpr int OFF_META = NSTAGE * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_META + NSTAGE * (int)sizeof(TileMeta);
  static constexpr int OFF_SCORES = OFF_BAR + 2 * NSTAGE * 8;
  static constexpr int OFF_P = OFF_SCORES + G * kTile * 4;
  static constexpr int OFF_ALPHA = OFF_P + kTile * G * 4;
  static constexpr int OFF_RED = OFF_ALPHA + ((G * 4 + 15) / 16) * 16;
  static constexpr int OFF_HEADS = OFF_RED + NCW * G * D * 4;
  static size_t smem_bytes(int nh) {
    // head_off (i64), page_off (i32), len, n, r (i32), scales (2 x f32), per head
    return 128 + OFF_HEADS + (size_t)(nh + 1) * 8 + (size_t)(nh + 1) * 4 + (size_t)nh * 4 * 3 +
           (size_t)nh * 8 + 64;
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

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(128) : "memory");
}

// Barrier over the 128 consumer threads that also ORs a flag across them, so
// that a failed wait makes every consumer leave the loop together.
__device__ __forceinline__ bool consumer_sync_any(bool x) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q;\n"
      "  setp.ne.u32 p, %1, 0;\n"
      "  bar.red.or.pred q, 1, 128, p;\n"
      "  selp.u32 %0, 1, 0, q; }"
      : "=r"(r) : "r"((uint32_t)x) : "memory");
  return r != 0;
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

// 16 bytes of K or V -> EPC floats as float2 pairs
template <bool FP8>
__device__ __forceinline__ void unpack16(const uint4 x, float2* f) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  if constexpr (FP8) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] = e4m3x2_to_f32x2((uint16_t)(w[j] & 0xFFFF));
      f[2 * j + 1] = e4m3x2_to_f32x2((uint16_t)(w[j] >> 16));
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) f[j] = make_float2(bf16lo_to_f32(w[j]), bf16hi_to_f32(w[j]));
  }
}

template <class T>
__global__ void __launch_bounds__(T::NT)
k_decode_split(CacheView c, DecodeWork w, int layer, int batch, const uint16_t* __restrict__ q,
               int n_launch) {
  constexpr int D = T::D, G = T::G, RB = T::RB, CPR = T::CPR, EPC = T::EPC, NC = T::NC,
                RPP = T::RPP, NSTAGE = T::NSTAGE, NCW = T::NCW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  TileMeta* meta = reinterpret_cast<TileMeta*>(smem + T::OFF_META);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  uint64_t* empty = full + NSTAGE;
  float* s_scores = reinterpret_cast<float*>(smem + T::OFF_SCORES);   // [G][64]
  float* s_p = reinterpret_cast<float*>(smem + T::OFF_P);             // [64][G]
  float* s_alpha = reinterpret_cast<float*>(smem + T::OFF_ALPHA);     // [G]
  float* s_red = reinterpret_cast<float*>(smem + T::OFF_RED);         // [NCW][G][D]
  const int NH = batch * c.Hkv;
  long long* head_off = reinterpret_cast<long long*>(smem + T::OFF_HEADS);   // [NH + 1]
  int* page_off = reinterpret_cast<int*>(head_off + NH + 1);                 // [NH + 1]
  int* s_len = page_off + NH + 1;
  int* s_n = s_len + NH;
  int* s_r = s_n + NH;
  float* s_hscale = reinterpret_cast<float*>(s_r + NH);                      // [NH][2]

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long hi0 = (long long)layer * c.Bmax * c.Hkv;   // first head of this layer

  // ---- 1. units and pages of every head of the call; exclusive prefix
  {
    const int per = (NH + T::NT - 1) / T::NT;
    const int h0 = tid * per, h1 = min(NH, h0 + per);
    long long su = 0;
    int sp = 0;
    for (int h = h0; h < h1; ++h) {
      const int len = c.store_len[hi0 + h], n = c.tok_n[hi0 + h], r = c.tok_r[hi0 + h];
      s_len[h] = len;
      s_n[h] = n;
      s_r[h] = r;
      if (T::FP8) {
        s_hscale[2 * h] = c.head_scale[(hi0 + h) * 2];
        s_hscale[2 * h + 1] = c.head_scale[(hi0 + h) * 2 + 1];
      }
      su += len + (n - r);
      sp += (len + kTile - 1) / kTile + (n - r + kTile - 1) / kTile;
    }
    // block exclusive scan of (su, sp)
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
    long long bu = 0;
    int bp = 0;
    for (int i = 0; i < warp; ++i) { bu += s_wu[i]; bp += s_wp[i]; }
    long long eu = bu + iu - su;
    int ep = bp + ip - sp;
    for (int h = h0; h < h1; ++h) {
      head_off[h] = eu;
      page_off[h] = ep;
      const int len = s_len[h], live = s_n[h] - s_r[h];
      eu += len + live;
      ep += (len + kTile - 1) / kTile + (live + kTile - 1) / kTile;
    }
    if (tid == T::NT - 1) {
      head_off[NH] = eu;
      page_off[NH] = ep;
    }
    __syncthreads();
  }
  const long long total = head_off[NH];
  const long long want = (total + kMinUnitsPerCta - 1) / kMinUnitsPerCta;
  const int n_eff = (int)(want < n_launch ? (want > 0 ? want : 1) : n_launch);
  if (blockIdx.x == 0) {
    for (int h = tid; h <= NH; h += T::NT) w.head_off[h] = head_off[h];
    if (tid == 0) {
      *w.n_eff = n_eff;
      c.ctr->slots_decoded += (unsigned long long)total;   // one CTA, launches are ordered
      c.ctr->decode_calls += 1ull;
    }
  }
  if ((int)blockIdx.x >= n_eff || total == 0) return;
  const long long gs = (long long)blockIdx.x * total / n_eff;
  const long long ge = (long long)(blockIdx.x + 1) * total / n_eff;
  if (gs >= ge) return;

  // global page holding global unit x
  auto gpage = [&](long long x) -> int {
    const int h = upper_bound(head_off, NH + 1, x) - 1;
    const long long u = x - head_off[h];
    const int len = s_len[h];
    const int lp = u < len ? (int)(u / kTile) : (len + kTile - 1) / kTile + (int)((u - len) / kTile);
    return page_off[h] + lp;
  };
  const int gp_first = gpage(gs);
  const int ntiles = gpage(ge - 1) - gp_first + 1;

  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NC);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ================= producer: lane s owns stage s, tiles s, s + NSTAGE, ...
    if (lane < NSTAGE) {
      for (int i = lane; i < ntiles; i += NSTAGE) {
        const int gp = gp_first + i;
        const int hidx = upper_bound(page_off, NH + 1, gp) - 1;
        const int lp = gp - page_off[hidx];
        const int len = s_len[hidx], n = s_n[hidx], r = s_r[hidx];
        const int sp = (len + kTile - 1) / kTile;
        const long long hoff = head_off[hidx];
        const long long lo = gs > hoff ? gs - hoff : 0;
        const long long hi_u = ge - hoff;   // exclusive bound in head units
        const long long hi = hi0 + hidx;
        TileMeta mt;
        mt.hidx = hidx;
        mt.flags = (i == 0 || lp == 0 ? kFirst : 0) |
                   (i == ntiles - 1 || gp + 1 == page_off[hidx + 1] ? kLast : 0);
        const uint8_t *ksrc0, *vsrc0, *ksrc1 = nullptr, *vsrc1 = nullptr;
        int n0rows, n1rows = 0;
        if (lp < sp) {   // store page lp
          const long long u0 = max((long long)lp * kTile, lo);
          const long long u1 = min((long long)min((lp + 1) * kTile, len), hi_u);
          const int row0 = (int)(u0 - (long long)lp * kTile);
          mt.nrows = (int)(u1 - u0);
          const long long blk = c.block_table[hi * c.max_blocks + lp];
          if (T::FP8) {
            mt.ks = c.bt_scale[(hi * c.max_blocks + lp) * 2];
            mt.vs = c.bt_scale[(hi * c.max_blocks + lp) * 2 + 1];
          } else {
            mt.ks = mt.vs = 1.0f;
          }
          ksrc0 = block_k(c, blk) + (long long)row0 * RB;
          vsrc0 = block_v(c, blk) + (long long)row0 * RB;
          n0rows = mt.nrows;
        } else {         // ring page lp - sp: units len + 64 * (lp - sp) ...
          const int rp = lp - sp;
          const long long u0 = max((long long)len + (long long)rp * kTile, lo);
          const long long u1 = min((long long)len + min((rp + 1) * kTile, n - r), hi_u);
          mt.nrows = (int)(u1 - u0);
          mt.p0 = r + (int)(u0 - len);
          mt.thresh = n - c.W;
          mt.R = c.R;
          mt.keep_base = hi * c.Rpad;
          mt.flags |= kRing | (mt.p0 < mt.thresh ? kPending : 0);
          mt.ks = T::FP8 ? s_hscale[2 * hidx] : 1.0f;
          mt.vs = T::FP8 ? s_hscale[2 * hidx + 1] : 1.0f;
          const int slot0 = mt.p0 % c.R;
          n0rows = min(mt.nrows, c.R - slot0);
          n1rows = mt.nrows - n0rows;
          ksrc0 = ring_k(c, hi) + (long long)slot0 * RB;
          vsrc0 = ring_v(c, hi) + (long long)slot0 * RB;
          ksrc1 = ring_k(c, hi);
          vsrc1 = ring_v(c, hi);
        }
        const int s = lane;
        const int k = i / NSTAGE;
        if (k > 0 && !mbar_wait(&empty[s], (k - 1) & 1)) {
          latch_error(c.ctr, FDMS_ERR_DEVICE);
          break;
        }
        meta[s] = mt;
        uint8_t* kdst = smem + s * T::STAGE_BYTES;
        uint8_t* vdst = kdst + T::KV_BYTES;
        const bool first = (mt.flags & kFirst) != 0;
        const uint32_t bytes = 2u * mt.nrows * RB + (first ? (uint32_t)T::Q_BYTES : 0u);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(kdst, ksrc0, n0rows * RB, &full[s]);
        bulk_g2s(vdst, vsrc0, n0rows * RB, &full[s]);
        if (n1rows > 0) {
          bulk_g2s(kdst + n0rows * RB, ksrc1, n1rows * RB, &full[s]);
          bulk_g2s(vdst + n0rows * RB, vsrc1, n1rows * RB, &full[s]);
        }
        if (first) {
          const int b = hidx / c.Hkv, h = hidx % c.Hkv;
          const uint16_t* qsrc = q + ((long long)b * c.Hq + (long long)h * G) * D;
          bulk_g2s(vdst + T::KV_BYTES, qsrc, T::Q_BYTES, &full[s]);
        }
      }
    }
    return;
  }

  // ================= consumers
  const int ch = tid % CPR;   // chunk of a row this thread owns
  const int rs = tid / CPR;   // row subset
  const float qscale = c.softmax_scale * kLog2e;
  float2 qf[G][EPC / 2];
  float2 acc[G][EPC / 2];
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};   // softmax warps
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPC / 2; ++e) acc[g][e] = make_float2(0.f, 0.f);

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % NSTAGE;
    const bool ok = mbar_wait(&full[s], (i / NSTAGE) & 1);
    TileMeta mt = meta[s];
    if (!ok) {            // stage never filled: touch nothing of it
      mt.nrows = 0;
      mt.flags = 0;
    }
    const uint8_t* Ks = smem + s * T::STAGE_BYTES;
    const uint8_t* Vs = Ks + T::KV_BYTES;
    const uint16_t* Qs = reinterpret_cast<const uint16_t*>(Vs + T::KV_BYTES);
    const int nrows = mt.nrows;

    if (mt.flags & kFirst) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int v8 = 0; v8 < EPC / 8; ++v8) {   // q is bf16: 8 elements per 16 bytes
          const uint4 x = *reinterpret_cast<const uint4*>(Qs + g * D + ch * EPC + v8 * 8);
          float2 f[4];
          unpack16<false>(x, f);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            qf[g][v8 * 4 + j] = make_float2(f[j].x * qscale, f[j].y * qscale);
            acc[g][v8 * 4 + j] = make_float2(0.f, 0.f);
          }
        }
      }
      m_run[0] = m_run[1] = -INFINITY;
      l_run[0] = l_run[1] = 0.0f;
    }

    // ---- scores: rows rs, rs + RPP, ... of this page
    const bool pend = (mt.flags & kPending) != 0;
    for (int k0 = 0; k0 < nrows; k0 += RPP) {
      const int row = k0 + rs;
      const uint4 x = *reinterpret_cast<const uint4*>(Ks + row * RB + ch * 16);
      float2 kf[EPC / 2];
      unpack16<T::FP8>(x, kf);
      float sc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < EPC / 2; ++e) a = ffma2(qf[g][e], kf[e], a);
        sc[g] = a.x + a.y;
      }
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], off);
      if (ch == 0 && row < nrows) {
        bool vis = true;
        if (pend) {
          const int p = mt.p0 + row;
          if (p < mt.thresh) vis = c.ring_keep[mt.keep_base + p % mt.R] != 0;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) s_scores[g * kTile + row] = vis ? sc[g] * mt.ks : -INFINITY;
      }
    }
    if (consumer_sync_any(!ok)) {
      if (tid == 0) latch_error(c.ctr, FDMS_ERR_DEVICE);
      break;
    }

    // ---- online softmax, one warp per head (two heads per warp when G = 8)
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int g = warp + t * NCW;
      if (g < G) {
        const float s0 = lane < nrows ? s_scores[g * kTile + lane] : -INFINITY;
        const float s1 = lane + 32 < nrows ? s_scores[g * kTile + lane + 32] : -INFINITY;
        float mt_ = fmaxf(s0, s1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, off));
        const float mn = fmaxf(m_run[t], mt_);
        float p0 = 0.f, p1 = 0.f, al = 1.f;
        if (mn != -INFINITY) {
          p0 = fast_exp2(s0 - mn);
          p1 = fast_exp2(s1 - mn);
          al = fast_exp2(m_run[t] - mn);
        }
        float ls = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        l_run[t] = l_run[t] * al + ls;
        m_run[t] = mn;
        s_p[lane * G + g] = p0 * mt.vs;
        s_p[(lane + 32) * G + g] = p1 * mt.vs;
        if (lane == 0) s_alpha[g] = al;
      }
    }
    consumer_sync();

    // ---- o += p * v over the page's rows
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float a = s_alpha[g];
#pragma unroll
      for (int e = 0; e < EPC / 2; ++e) acc[g][e] = make_float2(acc[g][e].x * a, acc[g][e].y * a);
    }
    for (int k0 = 0; k0 < nrows; k0 += RPP) {
      const int row = k0 + rs;
      if (row < nrows) {
        const uint4 x = *reinterpret_cast<const uint4*>(Vs + row * RB + ch * 16);
        float2 vf[EPC / 2];
        unpack16<T::FP8>(x, vf);
        float p[G];
#pragma unroll
        for (int g = 0; g < G; ++g) p[g] = s_p[row * G + g];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < EPC / 2; ++e) acc[g][e] = ffma2(make_float2(p[g], p[g]), vf[e], acc[g][e]);
      }
    }
    mbar_arrive(&empty[s]);

    if (mt.flags & kLast) {
      // sum the row subsets: first inside the warp, then across the warps
#pragma unroll
      for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < EPC / 2; ++e) {
            acc[g][e].x += __shfl_xor_sync(0xffffffffu, acc[g][e].x, off);
            acc[g][e].y += __shfl_xor_sync(0xffffffffu, acc[g][e].y, off);
          }
      if (lane < CPR) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < EPC / 2; ++e)
            *reinterpret_cast<float2*>(&s_red[(warp * G + g) * D + ch * EPC + 2 * e]) = acc[g][e];
      }
      consumer_sync();
      const long long part = (long long)blockIdx.x + mt.hidx;
      for (int idx = tid; idx < G * D; idx += NC) {
        float sum = 0.f;
#pragma unroll
        for (int wv = 0; wv < NCW; ++wv) sum += s_red[wv * G * D + idx];
        w.part_o[part * G * D + idx] = sum;
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int g = warp + t * NCW;
        if (g < G && lane == 0) {
          w.part_ml[(part * G + g) * 2] = m_run[t];
          w.part_ml[(part * G + g) * 2 + 1] = l_run[t];
        }
      }
      consumer_sync();
    }
  }
}

// CTA of unit x under the split: the largest c with floor(c * T / N) <= x.
__device__ __forceinline__ int cta_of(long long x, long long total, int n) {
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
    const int c0 = cta_of(s, total, n), c1 = cta_of(e - 1, total, n);
    for (int cc = c0; cc <= c1; ++cc) {
      const long long part = (long long)cc + hidx;
      M = fmaxf(M, w.part_ml[(part * G + g) * 2]);
    }
    if (M != -INFINITY) {
      for (int cc = c0; cc <= c1; ++cc) {
        const long long part = (long long)cc + hidx;
        const float m = w.part_ml[(part * G + g) * 2];
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
      lse[(long long)b * Hq + qh] = (M == -INFINITY) ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
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
      cache->view, cache->work, layer, batch, static_cast<const uint16_t*>(q), cache->decode_ctas);
  return cudaGetLastError() == cudaSuccess ? FDMS_OK : FDMS_ERR_CUDA;
}

template <class T>
fdms_status setup_t(fdms_cache* cache) {
  const int nh = cache->view.Bmax * cache->view.Hkv;
  const size_t smem = T::smem_bytes(nh);
  if (cudaFuncSetAttribute(k_decode_split<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return FDMS_ERR_UNSUPPORTED;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode_split<T>, T::NT, smem) !=
          cudaSuccess || per_sm < 1)
    return FDMS_ERR_UNSUPPORTED;
  cache->ctas_per_sm = per_sm;
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
  w.max_parts = ctas + c.Bmax * c.Hkv;
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

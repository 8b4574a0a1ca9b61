// Host side of the C ABI: cache creation and teardown, counters, inspection.
//
// The cache is the compact KV store of FastDMS ("FastDMS: 6.4X KV-cache
// compression running faster than vLLM BF16/FP8", aiwitness.kr/community/
// 1t3vlrx: survivors of per-head DMS eviction kept in a store that physically
// reclaims dropped slots, plus a staging area), laid out for one B200:
//   - one shared pool of 64-slot blocks, K rows then V rows per block, handed
//     out by a device bump allocator, so a head's store grows block by block
//     and dropped tokens never take memory;
//   - per-(layer, seq, kv head) block tables, block scales and lengths;
//   - per-(layer, seq, kv head) rings of W + P - 1 slots: the staging area
//     that holds tokens until their keep decision is applied.
#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <vector>

#include "fdms_internal.cuh"

using namespace fdms;

namespace {

struct DeviceGuard {
  int prev = -1;   // the device to restore, or -1: none (it was already current)
  explicit DeviceGuard(int dev) {
    int cur = -1;
    if (cudaGetDevice(&cur) == cudaSuccess && cur == dev) return;
    prev = cur;
    cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

template <class T>
cudaError_t alloc(fdms_cache* c, T** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return cudaSuccess;
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, bytes);
  if (e != cudaSuccess) return e;
  if (!fdms_track(c, q, bytes)) return cudaErrorMemoryAllocation;
  *p = static_cast<T*>(q);
  return cudaSuccess;
}

void free_all(fdms_cache* c) {
  for (int i = 0; i < c->nallocs; ++i) cudaFree(c->allocs[i]);
  c->nallocs = 0;
  delete[] c->append_at;
  delete[] c->decode_at;
  delete[] c->tokens_since;
  delete[] c->decode_batch;
  delete[] c->decode_count;
  c->append_at = c->decode_at = c->tokens_since = c->decode_count = nullptr;
  c->decode_batch = nullptr;
}

bool valid_config(const fdms_config* cfg) {
  if (!cfg) return false;
  if (cfg->num_layers < 1 || cfg->max_batch < 1 || cfg->num_kv_heads < 1) return false;
  if (cfg->num_q_heads < 1 || cfg->num_q_heads % cfg->num_kv_heads != 0) return false;
  if (cfg->window < 0 || cfg->compact_period < 1 || cfg->max_seq_len < 1) return false;
  if (cfg->num_blocks < 0 || cfg->decode_ctas < 0) return false;
  if (cfg->kv_dtype != FDMS_KV_BF16 && cfg->kv_dtype != FDMS_KV_FP8_E4M3 &&
      cfg->kv_dtype != FDMS_KV_FP8_E4M3_BLOCK)
    return false;
  if (!(cfg->softmax_scale >= 0.0f) || !std::isfinite(cfg->softmax_scale)) return false;
  if ((long long)cfg->window + cfg->compact_period > (1LL << 30)) return false;
  return true;
}

bool supported_config(const fdms_config* cfg) {
  const int G = cfg->num_q_heads / cfg->num_kv_heads;
  if (cfg->head_dim != 64 && cfg->head_dim != 128) return false;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if ((long long)cfg->max_batch * cfg->num_kv_heads > 4096) return false;
  return true;
}

// Totals over all heads, one CTA (the stats call is not on the hot path).
__global__ void __launch_bounds__(1024) k_stats(CacheView c) {
  __shared__ unsigned long long s_tok[32], s_store[32], s_ring[32], s_seal[32];
  const long long heads = (long long)c.L * c.Bmax * c.Hkv;
  unsigned long long tok = 0, store = 0, ring = 0, seal = 0;
  for (long long hi = threadIdx.x; hi < heads; hi += blockDim.x) {
    const int n = c.tok_n[hi], r = c.tok_r[hi], len = c.store_len[hi];
    store += (unsigned long long)len;
    seal += (unsigned long long)(len / kBlockSlots * kBlockSlots);
    ring += (unsigned long long)(n - r);
    if (hi % c.Hkv == 0) tok += (unsigned long long)n;
  }
  for (int off = 16; off > 0; off >>= 1) {
    tok += __shfl_xor_sync(0xffffffffu, tok, off);
    store += __shfl_xor_sync(0xffffffffu, store, off);
    ring += __shfl_xor_sync(0xffffffffu, ring, off);
    seal += __shfl_xor_sync(0xffffffffu, seal, off);
  }
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  if (l == 0) { s_tok[w] = tok; s_store[w] = store; s_ring[w] = ring; s_seal[w] = seal; }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long a = 0, b = 0, d = 0, e = 0;
    for (int i = 0; i < (int)(blockDim.x / 32); ++i) {
      a += s_tok[i]; b += s_store[i]; d += s_ring[i]; e += s_seal[i];
    }
    c.ctr->tokens = a;
    c.ctr->slots_store = b;
    c.ctr->slots_ring = d;
    c.ctr->slots_sealed = e;
  }
}

// fdms_cache_read_head for per-block FP8: host rows of 2 D bytes; sealed
// entries carry their codes in the first D bytes and the block's scales, staged
// and ring entries their bf16 values and scale 0.
fdms_status read_head_block(const CacheView& v, long long hi, int n, int r, int len,
                            int32_t* pos_host, uint8_t* keep_host, void* k_host, void* v_host,
                            float* scale_host) {
  const int RB = v.RB, SRB = 2 * v.D;
  uint8_t* kh = static_cast<uint8_t*>(k_host);
  uint8_t* vh = static_cast<uint8_t*>(v_host);
  auto unswizzle = [](uint8_t* dst, const uint8_t* src, int rb, int row, bool is_v) {
    for (int b = 0; b < rb; b += 16) std::memcpy(dst + b, src + swz_byte(rb, is_v, row, b), 16);
  };
  cudaError_t e = cudaSuccess;
  const int nseal = len / kBlockSlots;
  std::vector<int32_t> bt(nseal > 0 ? nseal : 1);
  std::vector<float> bs(2 * (nseal > 0 ? nseal : 1));
  if (nseal > 0) {
    e = cudaMemcpy(bt.data(), v.block_table + hi * v.max_blocks, nseal * 4,
                   cudaMemcpyDeviceToHost);
    if (e == cudaSuccess)
      e = cudaMemcpy(bs.data(), v.bt_scale + hi * v.max_blocks * 2, nseal * 8,
                     cudaMemcpyDeviceToHost);
  }
  std::vector<uint8_t> tmp((size_t)kBlockSlots * SRB);
  for (int j = 0; j < nseal && e == cudaSuccess; ++j) {
    const int base = j * kBlockSlots;
    const long long blk = bt[j];
    for (int which = 0; which < 2 && e == cudaSuccess; ++which) {
      uint8_t* dst = which ? vh : kh;
      if (!dst) continue;
      e = cudaMemcpy(tmp.data(), which ? block_v(v, blk) : block_k(v, blk),
                     (size_t)kBlockSlots * RB, cudaMemcpyDeviceToHost);
      for (int i = 0; i < kBlockSlots; ++i) {
        uint8_t* row = dst + (size_t)(base + i) * SRB;
        std::memset(row, 0, SRB);
        unswizzle(row, tmp.data() + (size_t)i * RB, RB, i, which == 1);
      }
    }
    if (pos_host && e == cudaSuccess)
      e = cudaMemcpy(pos_host + base, v.blk_pos + blk * kBlockSlots, kBlockSlots * 4,
                     cudaMemcpyDeviceToHost);
    for (int i = 0; i < kBlockSlots; ++i) {
      if (keep_host) keep_host[base + i] = 1;
      if (scale_host) {
        scale_host[2 * (base + i)] = bs[2 * j];
        scale_host[2 * (base + i) + 1] = bs[2 * j + 1];
      }
    }
  }
  // staged rows: the store's partly filled block
  const int staged = len - nseal * kBlockSlots;
  if (staged > 0 && e == cudaSuccess) {
    const int base = nseal * kBlockSlots;
    for (int which = 0; which < 2 && e == cudaSuccess; ++which) {
      uint8_t* dst = which ? vh : kh;
      if (!dst) continue;
      e = cudaMemcpy(tmp.data(), which ? stage_v(v, hi) : stage_k(v, hi),
                     (size_t)staged * SRB, cudaMemcpyDeviceToHost);
      for (int i = 0; i < staged; ++i)
        unswizzle(dst + (size_t)(base + i) * SRB, tmp.data() + (size_t)i * SRB, SRB, i,
                  which == 1);
    }
    if (pos_host && e == cudaSuccess)
      e = cudaMemcpy(pos_host + base, v.stage_pos + hi * kBlockSlots, (size_t)staged * 4,
                     cudaMemcpyDeviceToHost);
    for (int i = 0; i < staged; ++i) {
      if (keep_host) keep_host[base + i] = 1;
      if (scale_host) scale_host[2 * (base + i)] = scale_host[2 * (base + i) + 1] = 0.0f;
    }
  }
  if (e != cudaSuccess) return FDMS_ERR_CUDA;
  // ring, in position order r..n-1, bf16
  if (n > r) {
    std::vector<uint8_t> rk((size_t)v.R * SRB), rv((size_t)v.R * SRB), rkeep(v.R);
    e = cudaMemcpy(rk.data(), ring_k(v, hi), rk.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(rv.data(), ring_v(v, hi), rv.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess)
      e = cudaMemcpy(rkeep.data(), v.ring_keep + hi * v.Rpad, v.R, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return FDMS_ERR_CUDA;
    for (int p = r; p < n; ++p) {
      const int slot = p % v.R, i = len + (p - r);
      if (pos_host) pos_host[i] = p;
      if (keep_host) keep_host[i] = rkeep[slot];
      if (kh) unswizzle(kh + (size_t)i * SRB, rk.data() + (size_t)slot * SRB, SRB, slot, false);
      if (vh) unswizzle(vh + (size_t)i * SRB, rv.data() + (size_t)slot * SRB, SRB, slot, true);
      if (scale_host) scale_host[2 * i] = scale_host[2 * i + 1] = 0.0f;
    }
  }
  return FDMS_OK;
}

}  // namespace

extern "C" {

const char* fdms_status_string(fdms_status s) {
  switch (s) {
    case FDMS_OK: return "ok";
    case FDMS_ERR_INVALID_ARG: return "invalid argument";
    case FDMS_ERR_OUT_OF_BLOCKS: return "block pool exhausted";
    case FDMS_ERR_CUDA: return "CUDA runtime error";
    case FDMS_ERR_UNSUPPORTED: return "unsupported configuration";
    case FDMS_ERR_DEVICE: return "device-detected error";
  }
  return "unknown status";
}

fdms_status fdms_cache_create(const fdms_config* cfg, int device, void* stream,
                              fdms_cache** out) {
  if (!out) return FDMS_ERR_INVALID_ARG;
  *out = nullptr;
  if (!valid_config(cfg)) return FDMS_ERR_INVALID_ARG;
  if (!supported_config(cfg)) return FDMS_ERR_UNSUPPORTED;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) return FDMS_ERR_CUDA;
  if (device < 0 || device >= ndev) return FDMS_ERR_INVALID_ARG;
  DeviceGuard guard(device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  fdms_cache* c = new fdms_cache();
  std::memset(c, 0, sizeof(*c));
  c->cfg = *cfg;
  c->device = device;
  c->append_at = new long long[cfg->num_layers]();
  c->decode_at = new long long[cfg->num_layers]();
  c->tokens_since = new long long[cfg->num_layers]();
  c->decode_batch = new int[cfg->num_layers]();
  c->decode_count = new long long[cfg->num_layers]();
  if (cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
    free_all(c);
    delete c;
    return FDMS_ERR_CUDA;
  }
  CacheView& v = c->view;
  v.L = cfg->num_layers;
  v.Bmax = cfg->max_batch;
  v.Hq = cfg->num_q_heads;
  v.Hkv = cfg->num_kv_heads;
  v.G = v.Hq / v.Hkv;
  v.D = cfg->head_dim;
  v.blk = cfg->kv_dtype == FDMS_KV_FP8_E4M3_BLOCK;
  v.fp8 = cfg->kv_dtype == FDMS_KV_FP8_E4M3 || v.blk;
  v.RB = v.D * (v.fp8 ? 1 : 2);
  v.RBR = v.blk ? 2 * v.D : v.RB;   // per-block FP8 stages its rows in bf16
  {
    const char* stall = std::getenv("FDMS_TEST_STALL_COPIES");
    v.stall_tx = (stall && stall[0] && std::strcmp(stall, "0") != 0) ? 16u : 0u;
  }
  v.W = cfg->window;
  v.P = cfg->compact_period;
  // ring capacity: W + P - 1 unresolved tokens at most, rounded up to whole
  // 64-slot pages so that ring pages line up with the store's page rows
  v.R = (v.W + v.P - 1 + kBlockSlots - 1) / kBlockSlots * kBlockSlots;
  v.Rpad = v.R;
  v.max_seq_len = cfg->max_seq_len;
  v.max_blocks = (cfg->max_seq_len + kBlockSlots - 1) / kBlockSlots;
  v.softmax_scale = cfg->softmax_scale > 0.0f ? cfg->softmax_scale
                                               : (float)(1.0 / std::sqrt((double)v.D));
  const long long heads = (long long)v.L * v.Bmax * v.Hkv;
  v.num_blocks = cfg->num_blocks > 0 ? cfg->num_blocks : heads * v.max_blocks;
  if (v.num_blocks >= (1LL << 31)) {
    free_all(c);
    delete c;
    return FDMS_ERR_INVALID_ARG;
  }

  cudaError_t e = cudaSuccess;
  auto A = [&](auto** p, size_t bytes) {
    if (e == cudaSuccess) e = alloc(c, p, bytes);
  };
  A(&v.pool, (size_t)v.num_blocks * 2 * kBlockSlots * v.RB);
  A(&v.blk_pos, (size_t)v.num_blocks * kBlockSlots * sizeof(int32_t));
  A(&v.block_table, (size_t)heads * v.max_blocks * sizeof(int32_t));
  A(&v.bt_scale, (size_t)heads * v.max_blocks * 2 * sizeof(float));
  A(&v.store_len, (size_t)heads * sizeof(int32_t));
  A(&v.tok_n, (size_t)heads * sizeof(int32_t));
  A(&v.tok_r, (size_t)heads * sizeof(int32_t));
  A(&v.ring, (size_t)heads * 2 * v.R * v.RBR);
  if (v.blk) {
    A(&v.stage, (size_t)heads * 2 * kBlockSlots * 2 * v.D);
    A(&v.stage_pos, (size_t)heads * kBlockSlots * sizeof(int32_t));
  }
  A(&v.ring_keep, (size_t)heads * v.Rpad);
  A(&v.head_scale, (size_t)heads * 2 * sizeof(float));
  A(&v.ctr, sizeof(DevCounters));
  if (e == cudaSuccess) {
    fdms_status st = fdms_decode_setup(c);   // sizes the split grid and its workspace
    if (st == FDMS_OK) st = fdms_append_setup(c);
    if (st != FDMS_OK) {
      free_all(c);
      delete c;
      return st;
    }
  }
  if (e == cudaSuccess) e = cudaMemsetAsync(v.store_len, 0, heads * sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(v.tok_n, 0, heads * sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(v.tok_r, 0, heads * sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(v.head_scale, 0, heads * 2 * sizeof(float), s);
  if (e == cudaSuccess && v.ring_keep) e = cudaMemsetAsync(v.ring_keep, 0, heads * v.Rpad, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(v.ctr, 0, sizeof(DevCounters), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    free_all(c);
    delete c;
    return FDMS_ERR_CUDA;
  }
  *out = c;
  return FDMS_OK;
}

fdms_status fdms_cache_destroy(fdms_cache* c) {
  if (!c) return FDMS_OK;
  DeviceGuard guard(c->device);
  cudaError_t e = cudaDeviceSynchronize();
  free_all(c);
  delete c;
  return e == cudaSuccess ? FDMS_OK : FDMS_ERR_CUDA;
}

fdms_status fdms_append_evict(fdms_cache* c, int layer, int batch, const int32_t* n_new_dev,
                              int max_new, const void* k_dev, const void* v_dev,
                              const uint8_t* keep_dev, const float* kv_scale_dev,
                              void* stream) {
  if (!c) return FDMS_ERR_INVALID_ARG;
  const CacheView& v = c->view;
  if (layer < 0 || layer >= v.L || batch < 0 || batch > v.Bmax || max_new < 0)
    return FDMS_ERR_INVALID_ARG;
  if (batch == 0 || max_new == 0) return FDMS_OK;
  if (!n_new_dev || !k_dev || !v_dev || !keep_dev) return FDMS_ERR_INVALID_ARG;
  if (((uintptr_t)k_dev | (uintptr_t)v_dev) & 15) return FDMS_ERR_INVALID_ARG;
  if (kv_scale_dev && (!v.fp8 || v.blk)) return FDMS_ERR_INVALID_ARG;
  if (max_new > v.max_seq_len) return FDMS_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  return fdms_launch_append(c, layer, batch, n_new_dev, max_new, k_dev, v_dev, keep_dev,
                            kv_scale_dev, static_cast<cudaStream_t>(stream));
}

fdms_status fdms_decode_attn(fdms_cache* c, int layer, int batch, const void* q_dev,
                             void* out_dev, void* stream) {
  if (!c) return FDMS_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->view.L || batch < 0 || batch > c->view.Bmax)
    return FDMS_ERR_INVALID_ARG;
  if (batch == 0) return FDMS_OK;
  if (!q_dev || !out_dev || (((uintptr_t)q_dev | (uintptr_t)out_dev) & 15))
    return FDMS_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  return fdms_launch_decode(c, layer, batch, q_dev, out_dev, 0, nullptr,
                            static_cast<cudaStream_t>(stream));
}

fdms_status fdms_decode_attn_f32(fdms_cache* c, int layer, int batch, const void* q_dev,
                                 float* out_dev, float* lse_dev, void* stream) {
  if (!c) return FDMS_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->view.L || batch < 0 || batch > c->view.Bmax)
    return FDMS_ERR_INVALID_ARG;
  if (batch == 0) return FDMS_OK;
  if (!q_dev || !out_dev || (((uintptr_t)q_dev | (uintptr_t)out_dev) & 15))
    return FDMS_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  return fdms_launch_decode(c, layer, batch, q_dev, out_dev, 1, lse_dev,
                            static_cast<cudaStream_t>(stream));
}

fdms_status fdms_cache_stats(fdms_cache* c, fdms_stats* out, void* stream) {
  if (!c || !out) return FDMS_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const CacheView& v = c->view;
  k_stats<<<1, 1024, 0, s>>>(v);
  DevCounters h;
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, v.ctr, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return FDMS_ERR_CUDA;
  const long long row = 2LL * v.RB;   // one K row + one V row
  const long long used = (long long)h.blocks_next < v.num_blocks ? (long long)h.blocks_next
                                                                 : v.num_blocks;
  std::memset(out, 0, sizeof(*out));
  out->tokens_appended = (long long)h.tokens;
  out->slots_store = (long long)h.slots_store;
  out->slots_ring = (long long)h.slots_ring;
  out->blocks_used = used;
  out->blocks_free = v.num_blocks - used;
  out->bytes_compact = (out->slots_store + out->slots_ring) * row;
  if (v.blk)   // sealed slots in E4M3, staged and ring slots in bf16
    out->bytes_compact = (long long)h.slots_sealed * row +
                         (out->slots_store - (long long)h.slots_sealed + out->slots_ring) * 2 * row;
  out->bytes_dense_equiv = out->tokens_appended * v.Hkv * row;
  out->bytes_reserved = (long long)c->bytes_reserved;
  out->fp8_saturations = (long long)h.saturations;
  out->slots_decoded = (long long)h.slots_decoded;
  out->decode_calls = (long long)h.decode_calls;
  out->bytes_decoded = (long long)h.bytes_decoded;
  out->error = h.error;
  return FDMS_OK;
}

fdms_status fdms_cache_read_head(fdms_cache* c, int layer, int seq, int kv_head, int capacity,
                                 int32_t* pos_host, uint8_t* keep_host, void* k_host,
                                 void* v_host, float* scale_host, fdms_head_info* info,
                                 void* stream) {
  if (!c || !info) return FDMS_ERR_INVALID_ARG;
  const CacheView& v = c->view;
  if (layer < 0 || layer >= v.L || seq < 0 || seq >= v.Bmax || kv_head < 0 ||
      kv_head >= v.Hkv || capacity < 0)
    return FDMS_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long hi = head_index(v, layer, seq, kv_head);
  int32_t n = 0, r = 0, len = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&n, v.tok_n + hi, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&r, v.tok_r + hi, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&len, v.store_len + hi, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return FDMS_ERR_CUDA;
  info->num_tokens = n;
  info->resolved = r;
  info->store_len = len;
  info->ring_len = n - r;
  const int total = len + (n - r);
  if (!pos_host && !keep_host && !k_host && !v_host && !scale_host) return FDMS_OK;
  if (capacity < total) return FDMS_ERR_INVALID_ARG;
  if (v.blk) return read_head_block(v, hi, n, r, len, pos_host, keep_host, k_host, v_host,
                                    scale_host);
  const int RB = v.RB;
  uint8_t* kh = static_cast<uint8_t*>(k_host);
  uint8_t* vh = static_cast<uint8_t*>(v_host);
  // compact store, block by block
  const int nblk = (len + kBlockSlots - 1) / kBlockSlots;
  std::vector<int32_t> bt(nblk > 0 ? nblk : 1);
  std::vector<float> bs(2 * (nblk > 0 ? nblk : 1));
  if (nblk > 0) {
    e = cudaMemcpy(bt.data(), v.block_table + hi * v.max_blocks, nblk * 4, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess)
      e = cudaMemcpy(bs.data(), v.bt_scale + hi * v.max_blocks * 2, nblk * 8,
                     cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return FDMS_ERR_CUDA;
  }
  std::vector<uint8_t> tmp((size_t)kBlockSlots * RB);
  auto unswizzle = [&](uint8_t* dst, const uint8_t* src, int row, bool is_v) {
    for (int b = 0; b < RB; b += 16) std::memcpy(dst + b, src + swz_byte(RB, is_v, row, b), 16);
  };
  for (int j = 0; j < nblk && e == cudaSuccess; ++j) {
    const int rows = (len - j * kBlockSlots) < kBlockSlots ? (len - j * kBlockSlots) : kBlockSlots;
    const int base = j * kBlockSlots;
    const long long blk = bt[j];
    if (kh) {
      e = cudaMemcpy(tmp.data(), block_k(v, blk), (size_t)rows * RB, cudaMemcpyDeviceToHost);
      for (int i = 0; i < rows; ++i)
        unswizzle(kh + (size_t)(base + i) * RB, tmp.data() + (size_t)i * RB, i, false);
    }
    if (vh && e == cudaSuccess) {
      e = cudaMemcpy(tmp.data(), block_v(v, blk), (size_t)rows * RB, cudaMemcpyDeviceToHost);
      for (int i = 0; i < rows; ++i)
        unswizzle(vh + (size_t)(base + i) * RB, tmp.data() + (size_t)i * RB, i, true);
    }
    if (pos_host && e == cudaSuccess)
      e = cudaMemcpy(pos_host + base, v.blk_pos + blk * kBlockSlots, (size_t)rows * 4,
                     cudaMemcpyDeviceToHost);
    for (int i = 0; i < rows; ++i) {
      if (keep_host) keep_host[base + i] = 1;
      if (scale_host) {
        scale_host[2 * (base + i)] = bs[2 * j];
        scale_host[2 * (base + i) + 1] = bs[2 * j + 1];
      }
    }
  }
  if (e != cudaSuccess) return FDMS_ERR_CUDA;
  // ring, in position order r..n-1 (position p sits in slot p % R)
  if (n > r) {
    std::vector<uint8_t> rk((size_t)v.R * RB), rv((size_t)v.R * RB), rkeep(v.R);
    float hs[2] = {1.0f, 1.0f};
    e = cudaMemcpy(rk.data(), ring_k(v, hi), rk.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(rv.data(), ring_v(v, hi), rv.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess)
      e = cudaMemcpy(rkeep.data(), v.ring_keep + hi * v.Rpad, v.R, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && v.fp8)
      e = cudaMemcpy(hs, v.head_scale + hi * 2, 8, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return FDMS_ERR_CUDA;
    for (int p = r; p < n; ++p) {
      const int slot = p % v.R, i = len + (p - r);
      if (pos_host) pos_host[i] = p;
      if (keep_host) keep_host[i] = rkeep[slot];
      if (kh) unswizzle(kh + (size_t)i * RB, rk.data() + (size_t)slot * RB, slot, false);
      if (vh) unswizzle(vh + (size_t)i * RB, rv.data() + (size_t)slot * RB, slot, true);
      if (scale_host) {
        scale_host[2 * i] = hs[0];
        scale_host[2 * i + 1] = hs[1];
      }
    }
  }
  return FDMS_OK;
}

}  // extern "C"

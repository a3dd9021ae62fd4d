// pool_kernels.cu -- KV commit into the dual pool and the window-safe prefix-match length.
//
// Rolling buffer: position t lives in slot t mod W ("Sliding Window Attention (SWA)
// no riron to jisso", section "Rolling Buffer KV Cache", eq. (7)). Paged pool: position
// t of a sequence lives in page page_table[t / page_size], row t mod page_size.
// Window-safe length: "MiMo v2.5 inference optimisation", section "KV cache redesign".
#include "common.cuh"
#include "internal.h"

namespace hswa {

// One thread moves 16 bytes (8 bf16). Rows are (sequence b, token t, KV head g) of d elements.
// FP8 pools: the 8 values are stored as E4M3(fp32(x) * fp32(1 / scale)) in 8 bytes, scale of
// (layer, g) for K and for V.
template <int D, bool FP8>
__global__ void __launch_bounds__(256) append_kernel(
    const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int n_seqs, int n_tok, int Hkv,
    const int64_t* __restrict__ start_pos, const int32_t* __restrict__ seq_ids,
    const int32_t* __restrict__ page_table, int pt_stride,
    uint8_t* __restrict__ dst_k, uint8_t* __restrict__ dst_v, int is_swa, int W, int n_swa, int layer,
    int max_seqs, int64_t pages, int page_size, const float* __restrict__ inv_k,
    const float* __restrict__ inv_v, int* err) {
  constexpr int VEC = 8;
  constexpr int PER_ROW = D / VEC;
  const int64_t rows = (int64_t)n_seqs * n_tok * Hkv;
  const int64_t total = rows * PER_ROW;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / PER_ROW;
    const int c = (int)(idx % PER_ROW);
    const int g = (int)(row % Hkv);
    const int64_t bt = row / Hkv;
    const int t = (int)(bt % n_tok);
    const int b = (int)(bt / n_tok);
    const int64_t pos = start_pos[b] + t;
    int64_t dst_row;
    if (is_swa) {
      if (t < n_tok - W) continue;  // overwritten later in the same chunk
      const int seq = seq_ids[b];
      if (seq < 0 || seq >= max_seqs || pos < 0) {
        record_error(err, HSWA_ERR_DEVICE_BOUNDS);
        continue;
      }
      dst_row = (((int64_t)seq * n_swa + layer) * Hkv + g) * W + (pos % W);
    } else {
      const int64_t lp = pos / page_size;
      if (pos < 0 || lp >= pt_stride) {
        record_error(err, HSWA_ERR_DEVICE_BOUNDS);
        continue;
      }
      const int32_t page = page_table[(int64_t)b * pt_stride + lp];
      if (page < 0 || page >= pages) {
        record_error(err, HSWA_ERR_DEVICE_BOUNDS);
        continue;
      }
      dst_row = (((int64_t)layer * pages + page) * Hkv + g) * page_size + (pos % page_size);
    }
    const uint4* src_k = reinterpret_cast<const uint4*>(k + row * D) + c;
    const uint4* src_v = reinterpret_cast<const uint4*>(v + row * D) + c;
    if constexpr (FP8) {
      const float ik = inv_k[g], iv = inv_v[g];
      const uint4 a = __ldg(src_k), b = __ldg(src_v);
      auto q8 = [](const uint4& x, float inv) {
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t o[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float f0 = __uint_as_float(w[2 * h] << 16) * inv, f1 = __uint_as_float(w[2 * h] & 0xFFFF0000u) * inv;
          const float f2 = __uint_as_float(w[2 * h + 1] << 16) * inv,
                      f3 = __uint_as_float(w[2 * h + 1] & 0xFFFF0000u) * inv;
          o[h] = (uint32_t)pack_e4m3x2(f0, f1) | ((uint32_t)pack_e4m3x2(f2, f3) << 16);
        }
        return make_uint2(o[0], o[1]);
      };
      reinterpret_cast<uint2*>(dst_k + dst_row * D)[c] = q8(a, ik);
      reinterpret_cast<uint2*>(dst_v + dst_row * D)[c] = q8(b, iv);
    } else {
      reinterpret_cast<uint4*>(dst_k + dst_row * D * 2)[c] = __ldg(src_k);
      reinterpret_cast<uint4*>(dst_v + dst_row * D * 2)[c] = __ldg(src_v);
    }
  }
}

int launch_append(const hswa_pool* pool, int layer, int n_seqs, const int32_t* seq_ids,
                  const int64_t* start_pos, int n_tok, const uint16_t* k, const uint16_t* v,
                  const int32_t* page_table, int pt_stride, cudaStream_t stream) {
  const hswa_pool_desc& D = pool->desc;
  const bool is_swa = layer < D.n_swa_layers;
  const int64_t total = (int64_t)n_seqs * n_tok * D.n_kv_heads * (D.head_dim / 8);
  if (total == 0) return HSWA_OK;
  const int sms = pool->sms;
  const int64_t want = (total + 255) / 256;
  const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
  uint8_t* dk = is_swa ? pool->ring_k8 : pool->page_k8;
  uint8_t* dv = is_swa ? pool->ring_v8 : pool->page_v8;
  const int l = is_swa ? layer : layer - D.n_swa_layers;
  const int n_layers = D.n_swa_layers + D.n_full_layers;
  const float* inv_k = pool->fp8 ? pool->scales + ((size_t)2 * n_layers + layer) * D.n_kv_heads : nullptr;
  const float* inv_v = pool->fp8 ? pool->scales + ((size_t)3 * n_layers + layer) * D.n_kv_heads : nullptr;
#define HSWA_APPEND(DD, F8)                                                                                    \
  append_kernel<DD, F8><<<grid, 256, 0, stream>>>(k, v, n_seqs, n_tok, D.n_kv_heads, start_pos, seq_ids,     \
                                                   page_table, pt_stride, dk, dv, is_swa, D.window,          \
                                                   D.n_swa_layers, l, D.max_seqs, D.pages_per_full_layer,     \
                                                   D.page_size, inv_k, inv_v, pool->err)
  if (D.head_dim == 128) {
    if (pool->fp8) HSWA_APPEND(128, true); else HSWA_APPEND(128, false);
  } else {
    if (pool->fp8) HSWA_APPEND(64, true); else HSWA_APPEND(64, false);
  }
#undef HSWA_APPEND
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("kv_pool_append: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

// Ring row dst of one sliding-window layer, slot by slot from the rows src[s]: one thread moves 16
// bytes of K and of V. Every ring keeps position p in slot p mod W, so a slot copied from another
// row keeps its position.
template <int ROW_BYTES>
__global__ void __launch_bounds__(256) gather_ring_kernel(uint8_t* __restrict__ ring_k, uint8_t* __restrict__ ring_v,
                                                          const int32_t* __restrict__ src, int W, int Hkv, int n_swa,
                                                          int layer, int max_seqs, int dst, int* err) {
  constexpr int PER_ROW = ROW_BYTES / 16;
  const int64_t total = (int64_t)W * Hkv * PER_ROW;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(idx % PER_ROW);
    const int64_t row = idx / PER_ROW;
    const int g = (int)(row % Hkv);
    const int slot = (int)(row / Hkv);
    const int sq = src[slot];
    if (sq < 0 || sq == dst) continue;
    if (sq >= max_seqs) {
      record_error(err, HSWA_ERR_DEVICE_BOUNDS);
      continue;
    }
    const int64_t from = ((((int64_t)sq * n_swa + layer) * Hkv + g) * W + slot) * ROW_BYTES;
    const int64_t to = ((((int64_t)dst * n_swa + layer) * Hkv + g) * W + slot) * ROW_BYTES;
    reinterpret_cast<uint4*>(ring_k + to)[c] = reinterpret_cast<const uint4*>(ring_k + from)[c];
    reinterpret_cast<uint4*>(ring_v + to)[c] = reinterpret_cast<const uint4*>(ring_v + from)[c];
  }
}

int launch_gather_ring(const hswa_pool* pool, int layer, int dst, const int32_t* src, cudaStream_t stream) {
  const hswa_pool_desc& D = pool->desc;
  const int row_bytes = D.head_dim * pool->esize;  // 64, 128 or 256
  const int64_t total = (int64_t)D.window * D.n_kv_heads * (row_bytes / 16);
  const int64_t want = (total + 255) / 256;
  const int grid = (int)(want < (int64_t)pool->sms * 8 ? want : (int64_t)pool->sms * 8);
#define HSWA_GATHER(RB)                                                                                    \
  gather_ring_kernel<RB><<<grid, 256, 0, stream>>>(pool->ring_k8, pool->ring_v8, src, D.window, D.n_kv_heads, \
                                                    D.n_swa_layers, layer, D.max_seqs, dst, pool->err)
  if (row_bytes == 256) HSWA_GATHER(256);
  else if (row_bytes == 128) HSWA_GATHER(128);
  else HSWA_GATHER(64);
#undef HSWA_GATHER
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("kv_pool_gather_ring: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

// Sliding window W = 1: row i attends only key i, whose softmax weight is exactly 1, so
// o_i = v_i of the query head's KV head (the W = 1 special case of "formal definition",
// eq. (5)). One thread moves 16 bytes of one (row, query head).
template <int D>
__global__ void __launch_bounds__(256) window1_kernel(const uint16_t* __restrict__ v, uint16_t* __restrict__ o,
                                                      int64_t rows, int Hq, int Hkv) {
  constexpr int PER = D / 8;
  const int G = Hq / Hkv;
  const int64_t total = rows * Hq * PER;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(idx % PER);
    const int64_t rh = idx / PER;
    const int h = (int)(rh % Hq);
    const int64_t row = rh / Hq;  // (batch, token)
    reinterpret_cast<uint4*>(o + rh * D)[c] =
        __ldg(reinterpret_cast<const uint4*>(v + (row * Hkv + h / G) * D) + c);
  }
}

int launch_window1(const hswa_pool* pool, const uint16_t* v, uint16_t* o, int B, int n_q, int Hq, int Hkv, int d,
                   cudaStream_t stream) {
  const int64_t rows = (int64_t)B * n_q;
  const int64_t total = rows * Hq * (d / 8);
  if (total == 0) return HSWA_OK;
  const int64_t want = (total + 255) / 256;
  const int grid = (int)(want < (int64_t)pool->sms * 16 ? want : (int64_t)pool->sms * 16);
  if (d == 128) window1_kernel<128><<<grid, 256, 0, stream>>>(v, o, rows, Hq, Hkv);
  else window1_kernel<64><<<grid, 256, 0, stream>>>(v, o, rows, Hq, Hkv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("swa_prefill_fwd: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

// One thread per request. With the ring holding positions [max(0, C-W), C):
//  * C > W: the only resumable lengths are 0 and C (every other tail reaches a
//    position older than C - W); C needs m >= C and all W slots valid.
//  * C <= W: slot s holds position s; L is safe iff L <= C and slots 0..L-1 are
//    valid, so the answer is min(m, C, first invalid slot).
__global__ void __launch_bounds__(128) window_safe_len_kernel(const int64_t* __restrict__ m,
                                                              const int64_t* __restrict__ c,
                                                              const uint32_t* __restrict__ valid, int W,
                                                              int n_req, int64_t* __restrict__ out) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= n_req) return;
  const int words = (W + 31) >> 5;
  const uint32_t* vr = valid + (int64_t)r * words;
  const int64_t M = m[r], C = c[r];
  int64_t res;
  if (M < 0 || C < 0) {
    res = 0;
  } else if (C > W) {
    bool all = true;
    for (int w = 0; w < words && all; ++w) {
      const int bits = (w == words - 1) ? (W - 32 * w) : 32;
      const uint32_t need = bits == 32 ? 0xFFFFFFFFu : ((1u << bits) - 1u);
      all = (__ldg(vr + w) & need) == need;
    }
    res = (all && M >= C) ? C : 0;
  } else {
    // first invalid slot among 0 .. C-1 (C <= W)
    int64_t first_bad = C;
    for (int w = 0; w * 32 < C; ++w) {
      const uint32_t inv = ~__ldg(vr + w);
      if (inv) {
        const int64_t s = 32 * (int64_t)w + (__ffs(inv) - 1);
        if (s < first_bad) first_bad = s;
        break;
      }
    }
    res = M < first_bad ? M : first_bad;
  }
  out[r] = res;
}

int launch_window_safe_len(const int64_t* m, const int64_t* c, const uint32_t* valid, int W, int n_req,
                           int64_t* out, cudaStream_t stream) {
  if (n_req == 0) return HSWA_OK;
  window_safe_len_kernel<<<(n_req + 127) / 128, 128, 0, stream>>>(m, c, valid, W, n_req, out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("window_safe_len: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

// One thread waits on a fresh mbarrier that nothing ever arrives at, through the same bounded
// wait every kernel of the library uses; the wait gives up after limit_ns and records
// HSWA_ERR_TIMEOUT in the error word, and the kernel returns normally.
__global__ void selftest_wait_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  (void)mbar_wait_limit(&bar, 0, err, limit_ns);
}

int launch_selftest_wait(int* err, uint64_t limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("hswa_selftest_wait_timeout: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

}  // namespace hswa

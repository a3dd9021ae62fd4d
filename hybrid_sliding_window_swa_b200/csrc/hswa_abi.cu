// hswa_abi.cu -- the C ABI of libhswa.so: argument validation, dual-pool carving,
// TMA descriptor encoding and dispatch to the kernels. No exception crosses the
// boundary; every call returns a status and leaves a message in hswa_last_error().
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <new>
#include <vector>

#include "internal.h"

namespace hswa {

static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

static bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box);

bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box);
}

bool make_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                  const uint32_t* box) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rank, dims, strides_bytes, box);
}

static bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides_bytes[i];
  }
  CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return false;
  }
  return true;
}

static size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

int check_device(const hswa_pool* pool, const char* who) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_error("%s: no current CUDA device: %s", who, cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  if (dev != pool->device) {
    set_error("%s: the pool lives on device %d but device %d is current", who, pool->device, dev);
    return HSWA_ERR_INVALID_ARG;
  }
  return HSWA_OK;
}

static int check_desc(const hswa_pool_desc* d) {
  if (!d) {
    set_error("null pool descriptor");
    return HSWA_ERR_INVALID_ARG;
  }
  if (d->n_swa_layers < 0 || d->n_full_layers < 0 || d->n_kv_heads < 1 || d->max_seqs < 0 ||
      d->pages_per_full_layer < 0) {
    set_error("invalid pool descriptor (negative count or zero KV heads)");
    return HSWA_ERR_INVALID_ARG;
  }
  if (d->kv_format != HSWA_KV_BF16 && d->kv_format != HSWA_KV_FP8_E4M3) {
    set_error("kv_format %d unknown (HSWA_KV_BF16 or HSWA_KV_FP8_E4M3)", d->kv_format);
    return HSWA_ERR_INVALID_ARG;
  }
  if (d->window < 1) {
    set_error("window must be >= 1 (got %d)", d->window);
    return HSWA_ERR_INVALID_ARG;
  }
  if (d->head_dim != 64 && d->head_dim != 128) {
    set_error("head_dim %d unsupported (64 or 128)", d->head_dim);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  if (d->page_size != 64) {
    set_error("page_size %d unsupported (64)", d->page_size);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  return HSWA_OK;
}

static int check_heads(const hswa_pool* pool, int n_q_heads) {
  const int hkv = pool->desc.n_kv_heads;
  if (n_q_heads < 1 || n_q_heads % hkv != 0 || n_q_heads / hkv > 16 || n_q_heads > 65535) {
    set_error("n_q_heads %d must be a positive multiple of n_kv_heads %d with ratio <= 16", n_q_heads, hkv);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  return HSWA_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// FP8 pools: [4][n_layers][Hkv] float32 scales, rounded up to 256 bytes; 0 for bf16 pools.
static size_t scale_bytes(const hswa_pool_desc* d) {
  if (d->kv_format != HSWA_KV_FP8_E4M3) return 0;
  return round256(4 * sizeof(float) * (size_t)(d->n_swa_layers + d->n_full_layers) * d->n_kv_heads);
}

}  // namespace hswa

using namespace hswa;

extern "C" {

const char* hswa_last_error(void) { return g_err; }

int kv_pool_layout(const hswa_pool_desc* desc, size_t* bytes_total, size_t* bytes_swa, size_t* bytes_full) {
  int rc = check_desc(desc);
  if (rc) return rc;
  const bool fp8 = desc->kv_format == HSWA_KV_FP8_E4M3;
  const size_t e = fp8 ? 1 : 2;
  const size_t swa = round256(2 * (size_t)desc->max_seqs * desc->n_swa_layers * desc->n_kv_heads *
                              (size_t)desc->window * desc->head_dim * e);
  const size_t full = round256(2 * (size_t)desc->n_full_layers * (size_t)desc->pages_per_full_layer *
                               desc->n_kv_heads * (size_t)desc->page_size * desc->head_dim * e);
  const size_t sc = scale_bytes(desc);
  if (bytes_swa) *bytes_swa = swa;
  if (bytes_full) *bytes_full = full;
  if (bytes_total) *bytes_total = swa + full + sc + 256;
  return HSWA_OK;
}

int kv_pool_create(const hswa_pool_desc* desc, void* dev_mem, size_t bytes, hswa_pool** out) {
  if (!out) {
    set_error("kv_pool_create: null output handle");
    return HSWA_ERR_INVALID_ARG;
  }
  *out = nullptr;
  size_t total = 0, swa = 0, full = 0;
  int rc = kv_pool_layout(desc, &total, &swa, &full);
  if (rc) return rc;
  const size_t sc_bytes = scale_bytes(desc);
  if (!dev_mem || (reinterpret_cast<uintptr_t>(dev_mem) & 255u) != 0) {
    set_error("kv_pool_create: device memory must be non-null and 256-byte aligned");
    return HSWA_ERR_INVALID_ARG;
  }
  if (bytes < total) {
    set_error("kv_pool_create: %zu bytes given, layout needs %zu", bytes, total);
    return HSWA_ERR_OUT_OF_MEMORY;
  }
  hswa_pool* p = new (std::nothrow) hswa_pool();
  if (!p) {
    set_error("kv_pool_create: host allocation failed");
    return HSWA_ERR_OUT_OF_MEMORY;
  }
  p->desc = *desc;
  cudaError_t de = cudaGetDevice(&p->device);
  if (de == cudaSuccess) de = cudaDeviceGetAttribute(&p->sms, cudaDevAttrMultiProcessorCount, p->device);
  if (de == cudaSuccess)
    de = cudaDeviceGetAttribute(&p->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device);
  if (de != cudaSuccess || p->sms < 1) {
    set_error("kv_pool_create: querying the current device failed: %s", cudaGetErrorString(de));
    delete p;
    return HSWA_ERR_CUDA;
  }
  p->base = static_cast<uint8_t*>(dev_mem);
  p->bytes_swa = swa;
  p->bytes_full = full;
  p->bytes_scales = sc_bytes;
  p->fp8 = desc->kv_format == HSWA_KV_FP8_E4M3;
  p->esize = p->fp8 ? 1 : 2;
  const size_t ring_half = (size_t)desc->max_seqs * desc->n_swa_layers * desc->n_kv_heads * (size_t)desc->window *
                           desc->head_dim * p->esize;  // bytes
  const size_t page_half = (size_t)desc->n_full_layers * (size_t)desc->pages_per_full_layer * desc->n_kv_heads *
                           (size_t)desc->page_size * desc->head_dim * p->esize;
  p->ring_k8 = p->base;
  p->ring_v8 = p->base + ring_half;
  p->page_k8 = p->base + swa;
  p->page_v8 = p->base + swa + page_half;
  p->ring_k = reinterpret_cast<uint16_t*>(p->ring_k8);
  p->ring_v = reinterpret_cast<uint16_t*>(p->ring_v8);
  p->page_k = reinterpret_cast<uint16_t*>(p->page_k8);
  p->page_v = reinterpret_cast<uint16_t*>(p->page_v8);
  p->scales = p->fp8 ? reinterpret_cast<float*>(p->base + swa + full) : nullptr;
  p->err = reinterpret_cast<int*>(p->base + swa + full + sc_bytes);
  const uint64_t D = desc->head_dim;
  p->ring_tma = false;
  const uint64_t ring_rows = (uint64_t)desc->max_seqs * desc->n_swa_layers * desc->n_kv_heads;
  if (!p->fp8 && desc->window % 128 == 0 && ring_rows > 0) {
    const uint64_t dims[3] = {D, (uint64_t)desc->window, ring_rows};
    const uint64_t strides[2] = {D * 2, (uint64_t)desc->window * D * 2};
    const uint32_t box[3] = {64, 128, 1};
    if (!make_tmap_bf16(&p->tm_ring_k, p->ring_k, 3, dims, strides, box) ||
        !make_tmap_bf16(&p->tm_ring_v, p->ring_v, 3, dims, strides, box)) {
      delete p;
      return HSWA_ERR_CUDA;
    }
    p->ring_tma = true;
  }
  p->page_tma = false;
  const uint64_t page_rows = (uint64_t)desc->n_full_layers * desc->pages_per_full_layer * desc->n_kv_heads;
  if (page_rows > 0x7FFFFFFFull) {
    set_error("kv_pool_create: too many (layer, page, head) rows for 32-bit coordinates");
    delete p;
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  if (!p->fp8 && page_rows > 0) {
    const uint64_t dims[3] = {D, (uint64_t)desc->page_size, page_rows};
    const uint64_t strides[2] = {D * 2, (uint64_t)desc->page_size * D * 2};
    const uint32_t box[3] = {64, 64, 1};
    if (!make_tmap_bf16(&p->tm_page_k, p->page_k, 3, dims, strides, box) ||
        !make_tmap_bf16(&p->tm_page_v, p->page_v, 3, dims, strides, box)) {
      delete p;
      return HSWA_ERR_CUDA;
    }
    p->page_tma = true;
  }
  p->page_tma8 = false;
  if (p->fp8 && page_rows > 0 && D == 128) {
    const uint64_t dims[3] = {D, (uint64_t)desc->page_size, page_rows};
    const uint64_t strides[2] = {D, (uint64_t)desc->page_size * D};
    const uint32_t box[3] = {128, 64, 1};
    if (!make_tmap_u8(&p->tm_page_k8, p->page_k8, 3, dims, strides, box) ||
        !make_tmap_u8(&p->tm_page_v8, p->page_v8, 3, dims, strides, box)) {
      delete p;
      return HSWA_ERR_CUDA;
    }
    p->page_tma8 = true;
  }
  cudaError_t e = cudaMemset(p->err, 0, 256);
  if (e == cudaSuccess && p->fp8) {
    // every scale 1 (and so every reciprocal 1)
    std::vector<float> ones(sc_bytes / sizeof(float), 1.0f);
    e = cudaMemcpy(p->scales, ones.data(), sc_bytes, cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    set_error("kv_pool_create: initialising the error word or the scales failed: %s", cudaGetErrorString(e));
    delete p;
    return HSWA_ERR_CUDA;
  }
  *out = p;
  return HSWA_OK;
}

int kv_pool_set_scales(hswa_pool* pool, int layer, const float* k_scale, const float* v_scale) {
  if (!pool || !k_scale || !v_scale) {
    set_error("kv_pool_set_scales: null argument");
    return HSWA_ERR_INVALID_ARG;
  }
  if (!pool->fp8) {
    set_error("kv_pool_set_scales: the pool stores bf16 entries; scales apply to FP8 pools");
    return HSWA_ERR_INVALID_ARG;
  }
  const hswa_pool_desc& D = pool->desc;
  const int n_layers = D.n_swa_layers + D.n_full_layers;
  if (layer < 0 || layer >= n_layers) {
    set_error("kv_pool_set_scales: layer %d out of range", layer);
    return HSWA_ERR_INVALID_ARG;
  }
  const int H = D.n_kv_heads;
  std::vector<float> v4(4 * (size_t)H);
  for (int g = 0; g < H; ++g) {
    if (!(k_scale[g] > 0.0f) || !(v_scale[g] > 0.0f) || !isfinite(k_scale[g]) || !isfinite(v_scale[g]) ||
        !isfinite(1.0f / k_scale[g]) || !isfinite(1.0f / v_scale[g])) {
      set_error("kv_pool_set_scales: scale of KV head %d must be finite and > 0 with a finite reciprocal", g);
      return HSWA_ERR_INVALID_ARG;
    }
    v4[g] = k_scale[g];
    v4[H + g] = v_scale[g];
    v4[2 * H + g] = 1.0f / k_scale[g];
    v4[3 * H + g] = 1.0f / v_scale[g];
  }
  if (int rc = check_device(pool, "kv_pool_set_scales")) return rc;
  for (int w = 0; w < 4; ++w) {
    cudaError_t e = cudaMemcpy(pool->scales + ((size_t)w * n_layers + layer) * H, v4.data() + (size_t)w * H,
                               sizeof(float) * H, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      set_error("kv_pool_set_scales: copy failed: %s", cudaGetErrorString(e));
      return HSWA_ERR_CUDA;
    }
  }
  return HSWA_OK;
}

int kv_pool_destroy(hswa_pool* pool) {
  delete pool;
  return HSWA_OK;
}

int kv_pool_append(hswa_pool* pool, int layer, int n_seqs, const int32_t* seq_ids, const int64_t* start_pos,
                   int n_tok, const hswa_bf16* k, const hswa_bf16* v, const int32_t* page_table, int pt_stride,
                   void* stream) {
  if (!pool) {
    set_error("kv_pool_append: null pool");
    return HSWA_ERR_INVALID_ARG;
  }
  const hswa_pool_desc& D = pool->desc;
  if (layer < 0 || layer >= D.n_swa_layers + D.n_full_layers) {
    set_error("kv_pool_append: layer %d out of range", layer);
    return HSWA_ERR_INVALID_ARG;
  }
  if (n_seqs < 0 || n_tok < 0) {
    set_error("kv_pool_append: negative sizes");
    return HSWA_ERR_INVALID_ARG;
  }
  if (int rc = check_device(pool, "kv_pool_append")) return rc;
  if (n_seqs == 0 || n_tok == 0) return HSWA_OK;
  const bool is_swa = layer < D.n_swa_layers;
  if (!k || !v || !start_pos || !aligned16(k) || !aligned16(v) || (is_swa && !seq_ids) ||
      (!is_swa && (!page_table || pt_stride < 1))) {
    set_error("kv_pool_append: missing or misaligned device pointer");
    return HSWA_ERR_INVALID_ARG;
  }
  return launch_append(pool, layer, n_seqs, seq_ids, start_pos, n_tok, k, v, page_table, pt_stride,
                       static_cast<cudaStream_t>(stream));
}

int kv_pool_gather_ring(hswa_pool* pool, int layer, int32_t dst_seq, const int32_t* src_seq, void* stream) {
  if (!pool) {
    set_error("kv_pool_gather_ring: null pool");
    return HSWA_ERR_INVALID_ARG;
  }
  const hswa_pool_desc& D = pool->desc;
  if (layer < 0 || layer >= D.n_swa_layers) {
    set_error("kv_pool_gather_ring: layer %d is not a sliding-window layer of this pool", layer);
    return HSWA_ERR_INVALID_ARG;
  }
  if (dst_seq < 0 || dst_seq >= D.max_seqs || !src_seq) {
    set_error("kv_pool_gather_ring: dst_seq %d outside [0, %d) or null src_seq", dst_seq, D.max_seqs);
    return HSWA_ERR_INVALID_ARG;
  }
  if (int rc = check_device(pool, "kv_pool_gather_ring")) return rc;
  return launch_gather_ring(pool, layer, dst_seq, src_seq, static_cast<cudaStream_t>(stream));
}

static int build_q_map(CUtensorMap* m, const void* base, int B, int n_q, int H, int d) {
  const uint64_t dims[4] = {(uint64_t)d, (uint64_t)H, (uint64_t)n_q, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)d * 2, (uint64_t)H * d * 2, (uint64_t)n_q * H * d * 2};
  const uint32_t box[4] = {64, 1, 128, 1};
  return make_tmap_bf16(m, base, 4, dims, strides, box) ? HSWA_OK : HSWA_ERR_CUDA;
}

// Output map: the epilogue of each warp stores its 32 rows of one 64-column half per box.
static int build_o_map(CUtensorMap* m, void* base, int B, int n_q, int H, int d) {
  const uint64_t dims[4] = {(uint64_t)d, (uint64_t)H, (uint64_t)n_q, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)d * 2, (uint64_t)H * d * 2, (uint64_t)n_q * H * d * 2};
  const uint32_t box[4] = {64, 1, 32, 1};
  return make_tmap_bf16(m, base, 4, dims, strides, box) ? HSWA_OK : HSWA_ERR_CUDA;
}

int swa_prefill_fwd(hswa_pool* pool, int layer, const hswa_bf16* q, const hswa_bf16* k, const hswa_bf16* v,
                    hswa_bf16* o, int B, int n_q, const int64_t* start_pos, const int32_t* seq_ids, int n_q_heads,
                    void* stream) {
  if (!pool) {
    set_error("swa_prefill_fwd: null pool");
    return HSWA_ERR_INVALID_ARG;
  }
  const hswa_pool_desc& D = pool->desc;
  if (layer < 0 || layer >= D.n_swa_layers) {
    set_error("swa_prefill_fwd: layer %d is not a sliding-window layer of this pool", layer);
    return HSWA_ERR_INVALID_ARG;
  }
  int rc = check_heads(pool, n_q_heads);
  if (rc) return rc;
  if ((rc = check_device(pool, "swa_prefill_fwd"))) return rc;
  if (B < 0 || n_q < 0 || B > 65535) {
    set_error("swa_prefill_fwd: bad B or n_q");
    return HSWA_ERR_INVALID_ARG;
  }
  if (B == 0 || n_q == 0) return HSWA_OK;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) {
    set_error("swa_prefill_fwd: missing or misaligned tensor pointer");
    return HSWA_ERR_INVALID_ARG;
  }
  if (start_pos && !seq_ids) {
    set_error("swa_prefill_fwd: seq_ids are required with start_pos");
    return HSWA_ERR_INVALID_ARG;
  }
  if (D.window == 1)  // the window is the diagonal alone: o_i = v_i
    return launch_window1(pool, v, o, B, n_q, n_q_heads, D.n_kv_heads, D.head_dim, static_cast<cudaStream_t>(stream));
  PrefillLaunch L{};
  L.B = B;
  L.n_q = n_q;
  L.Hq = n_q_heads;
  L.Hkv = D.n_kv_heads;
  L.d = D.head_dim;
  L.window = D.window;
  L.start_pos = start_pos;
  L.seq_ids = seq_ids;
  L.o = o;
  L.pool = pool;
  L.ring_layer = layer;
  L.layer = layer;
  if ((rc = build_q_map(&L.tm_q, q, B, n_q, n_q_heads, D.head_dim))) return rc;
  if ((rc = build_q_map(&L.tm_k, k, B, n_q, D.n_kv_heads, D.head_dim))) return rc;
  if ((rc = build_q_map(&L.tm_v, v, B, n_q, D.n_kv_heads, D.head_dim))) return rc;
  if ((rc = build_o_map(&L.tm_o, o, B, n_q, n_q_heads, D.head_dim))) return rc;
  return launch_prefill(L, static_cast<cudaStream_t>(stream));
}

int full_prefill_fwd(hswa_pool* pool, int layer, const hswa_bf16* q, hswa_bf16* o, int B, int n_q,
                     const int64_t* start_pos, const int32_t* page_table, int pt_stride, int n_q_heads,
                     void* stream) {
  if (!pool) {
    set_error("full_prefill_fwd: null pool");
    return HSWA_ERR_INVALID_ARG;
  }
  const hswa_pool_desc& D = pool->desc;
  if (layer < D.n_swa_layers || layer >= D.n_swa_layers + D.n_full_layers) {
    set_error("full_prefill_fwd: layer %d is not a full layer of this pool", layer);
    return HSWA_ERR_INVALID_ARG;
  }
  int rc = check_heads(pool, n_q_heads);
  if (rc) return rc;
  if ((rc = check_device(pool, "full_prefill_fwd"))) return rc;
  if (pool->fp8 && D.head_dim != 128) {
    set_error("full_prefill_fwd: FP8 pages are read with head_dim 128 only");
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  if (B < 0 || n_q < 0 || B > 65535) {
    set_error("full_prefill_fwd: bad B or n_q");
    return HSWA_ERR_INVALID_ARG;
  }
  if (B == 0 || n_q == 0) return HSWA_OK;
  if (!q || !o || !aligned16(q) || !aligned16(o) || !page_table || pt_stride < 1 ||
      !(pool->fp8 ? pool->page_tma8 : pool->page_tma)) {
    set_error("full_prefill_fwd: missing tensor pointer, page table, or pool pages");
    return HSWA_ERR_INVALID_ARG;
  }
  PrefillLaunch L{};
  L.B = B;
  L.n_q = n_q;
  L.Hq = n_q_heads;
  L.Hkv = D.n_kv_heads;
  L.d = D.head_dim;
  L.window = 0;
  L.start_pos = start_pos;
  L.page_table = page_table;
  L.pt_stride = pt_stride;
  L.o = o;
  L.pool = pool;
  L.full_layer = layer - D.n_swa_layers;
  L.layer = layer;
  if ((rc = build_q_map(&L.tm_q, q, B, n_q, n_q_heads, D.head_dim))) return rc;
  L.tm_k = pool->fp8 ? pool->tm_page_k8 : pool->tm_page_k;
  L.tm_v = pool->fp8 ? pool->tm_page_v8 : pool->tm_page_v;
  if ((rc = build_o_map(&L.tm_o, o, B, n_q, n_q_heads, D.head_dim))) return rc;
  return launch_prefill(L, static_cast<cudaStream_t>(stream));
}

int hybrid_decode_workspace_size(const hswa_pool* pool, int n_seqs, int n_q_per_seq, int n_q_heads,
                                 int64_t max_ctx_len, size_t* bytes) {
  if (!pool || !bytes || n_seqs < 0 || n_q_per_seq < 1 || n_q_per_seq > 8 || max_ctx_len < 0) {
    set_error("hybrid_decode_workspace_size: bad arguments");
    return HSWA_ERR_INVALID_ARG;
  }
  int rc = check_heads(pool, n_q_heads);
  if (rc) return rc;
  const hswa_pool_desc& D = pool->desc;
  // sized for a full layer, the larger of the two layer kinds
  *bytes = decode_workspace_bytes(n_seqs, n_q_per_seq, n_q_heads, D.n_kv_heads, D.head_dim, 0, max_ctx_len);
  return HSWA_OK;
}

}  // extern "C"

namespace hswa {

int prepare_decode(hswa_pool* pool, const char* who, int layer, const uint16_t* q, const uint16_t* k_new,
                   const uint16_t* v_new, uint16_t* o, int n_seqs, int n_q_per_seq, const int64_t* ctx_len,
                   int64_t max_ctx_len, const int32_t* seq_ids, const int32_t* page_table, int pt_stride,
                   int n_q_heads, DecodeLaunch* L, size_t* need) {
  if (!pool) {
    set_error("%s: null pool", who);
    return HSWA_ERR_INVALID_ARG;
  }
  const hswa_pool_desc& D = pool->desc;
  if (layer < 0 || layer >= D.n_swa_layers + D.n_full_layers) {
    set_error("%s: layer %d out of range", who, layer);
    return HSWA_ERR_INVALID_ARG;
  }
  int rc = check_heads(pool, n_q_heads);
  if (rc) return rc;
  if (n_seqs < 0 || n_q_per_seq < 1 || n_q_per_seq > 8 || max_ctx_len < 0) {
    set_error("%s: bad sizes (n_q_per_seq must be 1..8)", who);
    return HSWA_ERR_INVALID_ARG;
  }
  if (max_ctx_len > 0x7fffffffLL - 4096) {
    set_error("%s: positions must stay below 2^31", who);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  const int rows = n_q_per_seq * (n_q_heads / D.n_kv_heads);
  if (rows > 32) {
    set_error("%s: n_q_per_seq * (n_q_heads / n_kv_heads) = %d rows per KV head; at most 32 supported", who, rows);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  if ((rc = check_device(pool, who))) return rc;
  *L = DecodeLaunch{};
  *need = 0;
  if (n_seqs == 0) return HSWA_OK;
  const bool is_swa = layer < D.n_swa_layers;
  if (!q || !k_new || !v_new || !o || !ctx_len || !aligned16(q) || !aligned16(k_new) || !aligned16(v_new) ||
      !aligned16(o) || (is_swa && !seq_ids) || (!is_swa && (!page_table || pt_stride < 1))) {
    set_error("%s: missing or misaligned device pointer", who);
    return HSWA_ERR_INVALID_ARG;
  }
  const int window = is_swa ? D.window : 0;
  const size_t msm = decode_merge_smem_bytes(n_seqs, n_q_per_seq, n_q_heads, D.n_kv_heads, window, max_ctx_len);
  if (msm > (size_t)pool->smem_optin) {
    set_error("%s: max_ctx_len %lld gives %zu bytes of split-merge shared memory; this device allows %d", who,
              (long long)max_ctx_len, msm, pool->smem_optin);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  *need = decode_workspace_bytes(n_seqs, n_q_per_seq, n_q_heads, D.n_kv_heads, D.head_dim, window, max_ctx_len);
  L->n_seqs = n_seqs;
  L->layer = layer;
  L->n_qt = n_q_per_seq;
  L->Hq = n_q_heads;
  L->Hkv = D.n_kv_heads;
  L->d = D.head_dim;
  L->window = window;
  L->q = q;
  L->k_new = k_new;
  L->v_new = v_new;
  L->o = o;
  L->ctx_len = ctx_len;
  L->max_ctx_len = max_ctx_len;
  L->seq_ids = seq_ids;
  L->page_table = page_table;
  L->pt_stride = pt_stride;
  L->pool = pool;
  L->ring_layer = is_swa ? layer : 0;
  L->full_layer = is_swa ? 0 : layer - D.n_swa_layers;
  return HSWA_OK;
}

}  // namespace hswa

extern "C" {

int hybrid_decode_fwd(hswa_pool* pool, int layer, const hswa_bf16* q, const hswa_bf16* k_new,
                      const hswa_bf16* v_new, hswa_bf16* o, int n_seqs, int n_q_per_seq, const int64_t* ctx_len,
                      int64_t max_ctx_len, const int32_t* seq_ids, const int32_t* page_table, int pt_stride,
                      int n_q_heads, void* workspace, size_t ws_bytes, void* stream) {
  DecodeLaunch L;
  size_t need = 0;
  int rc = prepare_decode(pool, "hybrid_decode_fwd", layer, q, k_new, v_new, o, n_seqs, n_q_per_seq, ctx_len,
                          max_ctx_len, seq_ids, page_table, pt_stride, n_q_heads, &L, &need);
  if (rc || L.n_seqs == 0) return rc;
  if (ws_bytes < need || (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)))) {
    set_error("hybrid_decode_fwd: workspace of %zu bytes (256-aligned) needed, %zu given", need, ws_bytes);
    return HSWA_ERR_INVALID_ARG;
  }
  L.workspace = workspace;
  L.ws_bytes = ws_bytes;
  return launch_decode(L, static_cast<cudaStream_t>(stream));
}

int window_safe_len(const int64_t* match_len, const int64_t* cached_len, const uint32_t* slot_valid, int32_t W,
                    int32_t n_req, int64_t* out_len, void* stream) {
  if (W < 1 || n_req < 0) {
    set_error("window_safe_len: W must be >= 1 and n_req >= 0");
    return HSWA_ERR_INVALID_ARG;
  }
  if (n_req == 0) return HSWA_OK;
  if (!match_len || !cached_len || !slot_valid || !out_len) {
    set_error("window_safe_len: null device pointer");
    return HSWA_ERR_INVALID_ARG;
  }
  return launch_window_safe_len(match_len, cached_len, slot_valid, W, n_req, out_len,
                                static_cast<cudaStream_t>(stream));
}

int hswa_selftest_wait_timeout(hswa_pool* pool, int64_t limit_ns, void* stream) {
  if (!pool || limit_ns < 1000000 || limit_ns > 2000000000) {
    set_error("hswa_selftest_wait_timeout: a pool and a limit of 1 ms .. 2 s are required");
    return HSWA_ERR_INVALID_ARG;
  }
  if (int rc = check_device(pool, "hswa_selftest_wait_timeout")) return rc;
  return launch_selftest_wait(pool->err, (uint64_t)limit_ns, static_cast<cudaStream_t>(stream));
}

int hswa_pool_check_error(hswa_pool* pool, int* device_code) {
  if (!pool || !device_code) {
    set_error("hswa_pool_check_error: null argument");
    return HSWA_ERR_INVALID_ARG;
  }
  if (int rc = check_device(pool, "hswa_pool_check_error")) return rc;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    set_error("hswa_pool_check_error: device synchronisation failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  int code = 0;
  e = cudaMemcpy(&code, pool->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(pool->err, 0, sizeof(int));
  if (e != cudaSuccess) {
    set_error("hswa_pool_check_error: reading the error word failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  *device_code = code;
  return HSWA_OK;
}

}  // extern "C"

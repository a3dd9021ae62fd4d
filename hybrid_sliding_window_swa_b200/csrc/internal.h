// internal.h -- host-side pool object and kernel launch interfaces of libhswa.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hswa.h"

struct hswa_pool {
  hswa_pool_desc desc;
  int device;        // the CUDA device current at kv_pool_create; every call must run with it current
  int sms;           // its multiprocessor count
  int smem_optin;    // its largest opt-in shared memory per block (bytes)
  uint8_t* base;
  size_t bytes_swa, bytes_full, bytes_scales;
  bool fp8;          // entries are FP8 E4M3 codes (1 byte) instead of bf16 (2 bytes)
  int esize;         // bytes per element
  // element arrays (uint16_t for bf16 pools; for FP8 pools the same addresses hold bytes, see *8)
  uint16_t* ring_k;  // [max_seqs][n_swa][Hkv][W][d]
  uint16_t* ring_v;
  uint16_t* page_k;  // [n_full][pages][Hkv][page_size][d]
  uint16_t* page_v;
  uint8_t* ring_k8;  // the same regions as bytes
  uint8_t* ring_v8;
  uint8_t* page_k8;
  uint8_t* page_v8;
  float* scales;     // FP8: [4][n_layers][Hkv] = K scale, V scale, 1/K scale, 1/V scale (device)
  int* err;          // device error word
  bool ring_tma;     // W is a multiple of 128: ring tiles can be fetched with one TMA box
  CUtensorMap tm_ring_k, tm_ring_v;
  bool page_tma;
  CUtensorMap tm_page_k, tm_page_v;
  bool page_tma8;                     // FP8 pools with head_dim 128: pages as byte tiles
  CUtensorMap tm_page_k8, tm_page_v8; // [page_rows][64][128] bytes, 64-row boxes, 128-byte swizzle
};

namespace hswa {

// Thread-local error message of the ABI layer.
void set_error(const char* fmt, ...);

// HSWA_OK when the calling thread's current CUDA device is the pool's device; otherwise
// HSWA_ERR_INVALID_ARG with a message naming `who` (nothing may be launched for the call).
int check_device(const hswa_pool* pool, const char* who);

// Encode a 2-5 dimensional bf16 tiled tensor map with 128-byte swizzle.
// dims/strides: innermost first; strides in bytes for dims 1.. (dim 0 is contiguous).
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box);
// The same for 1-byte elements (FP8 codes), 128-byte swizzle.
bool make_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                  const uint32_t* box);

int launch_append(const hswa_pool* pool, int layer, int n_seqs, const int32_t* seq_ids,
                  const int64_t* start_pos, int n_tok, const uint16_t* k, const uint16_t* v,
                  const int32_t* page_table, int pt_stride, cudaStream_t stream);

int launch_gather_ring(const hswa_pool* pool, int layer, int dst, const int32_t* src, cudaStream_t stream);

int launch_selftest_wait(int* err, uint64_t limit_ns, cudaStream_t stream);

// Sliding window W = 1: o = v of each query head's KV head (k, q and the ring are not read).
int launch_window1(const hswa_pool* pool, const uint16_t* v, uint16_t* o, int B, int n_q, int Hq, int Hkv, int d,
                   cudaStream_t stream);

int launch_window_safe_len(const int64_t* m, const int64_t* c, const uint32_t* valid, int W, int n_req,
                           int64_t* out, cudaStream_t stream);

struct PrefillLaunch {
  // problem
  int B, n_q, Hq, Hkv, d;
  int window;  // >= 1 for SWA, 0 for full causal
  const int64_t* start_pos;  // device, may be null (all zero)
  const int32_t* seq_ids;    // SWA ring rows
  const int32_t* page_table; // full layers
  int pt_stride;
  uint16_t* o;
  // pool
  const hswa_pool* pool;
  int ring_layer;      // SWA layer index within the ring (SWA)
  int full_layer;      // full layer index within the paged pool (full)
  int layer;           // pool layer index (selects the FP8 scales)
  // tensor maps built by the ABI layer
  CUtensorMap tm_q, tm_k, tm_v;  // tm_k/tm_v: chunk K/V (SWA) or pages (full)
  CUtensorMap tm_o;              // output, stored 32 rows x 64 columns per TMA box
};

int launch_prefill(const PrefillLaunch& L, cudaStream_t stream);
// Sliding-window prefill with 1 <= W <= 129 (the band of a query tile spans at most two key tiles).
int launch_prefill_narrow(const PrefillLaunch& L, cudaStream_t stream);

struct DecodeLaunch {
  int n_seqs, n_qt, Hq, Hkv, d;
  int layer;   // pool layer index (selects the FP8 scales)
  int window;  // >= 1 SWA (ring), 0 full (pages)
  const uint16_t* q;
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t* o;
  const int64_t* ctx_len;
  int64_t max_ctx_len;
  const int32_t* seq_ids;
  const int32_t* page_table;
  int pt_stride;
  const hswa_pool* pool;
  int ring_layer, full_layer;
  void* workspace;
  size_t ws_bytes;
};

size_t decode_workspace_bytes(int n_seqs, int n_qt, int Hq, int Hkv, int d, int window, int64_t max_ctx_len);
// Dynamic shared memory of the split merge for these arguments (0 when no sequence can have two splits).
size_t decode_merge_smem_bytes(int n_seqs, int n_qt, int Hq, int Hkv, int window, int64_t max_ctx_len);

// Argument checks shared by hybrid_decode_fwd and hybrid_decode_fwd_noalloc (messages name `who`).
// On HSWA_OK, *L is filled except for workspace/ws_bytes and *need is the scratch the call uses;
// L->n_seqs == 0 means there is nothing to launch.
int prepare_decode(hswa_pool* pool, const char* who, int layer, const uint16_t* q, const uint16_t* k_new,
                   const uint16_t* v_new, uint16_t* o, int n_seqs, int n_q_per_seq, const int64_t* ctx_len,
                   int64_t max_ctx_len, const int32_t* seq_ids, const int32_t* page_table, int pt_stride,
                   int n_q_heads, DecodeLaunch* L, size_t* need);
int launch_decode(const DecodeLaunch& L, cudaStream_t stream);

}  // namespace hswa

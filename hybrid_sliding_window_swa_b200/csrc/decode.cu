// decode.cu -- one decode step of hybrid sliding-window attention, split over the KV
// sequence ("split-KV"), plus the log-sum-exp merge of the splits.
//
// Each sequence brings n_qt new query tokens at positions L .. L+n_qt-1 (one token and
// its multi-token-prediction drafts; "MiMo v2.5 inference optimisation", sections
// "architecture" and "KV cache redesign"). Draft t attends the cached keys in its window
// plus new tokens 0..t. Sliding-window layers read cached keys from the rolling buffer
// (slot = pos mod W, "Sliding Window Attention (SWA) no riron to jisso", section
// "Rolling Buffer KV Cache", eq. (7)); full layers read them through the page table.
//
// Work item = (sequence s, split c, KV head g): keys [klo + c*SPLIT, klo + (c+1)*SPLIT)
// of the cached range, plus the new tokens in the sequence's last split. The rows of an
// item are the n_qt * G query rows (token t, query head g*G + hh) that share KV head g,
// so every K/V byte is read from HBM once per step. A CTA of 4 warps streams 64-key
// blocks of K and V through a 3-stage cp.async pipeline; each warp takes 16 keys of a
// block, computes S = Q K^T and O += P V with mma.sync (bf16 in, fp32 accumulate), and
// keeps its own online-softmax state; the 4 warp states are merged through shared
// memory at the end of the item. The CTAs take items in the order plan_kernel builds (length
// buckets and longest first, see PlanView). Items with one split write the output directly; the
// others write (m, l, O) partials that merge_kernel combines:
//   o = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c,  M = max_c m_c.
#include <cstddef>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace hswa {

namespace {

constexpr int DEC_THREADS = 128;
constexpr int KB = 64;          // keys per block
constexpr int NST = 3;          // pipeline stages (bf16 blocks)
constexpr int NST8 = 6;         // pipeline stages (FP8 blocks: half the bytes, the same bytes in flight)
#ifndef HSWA_DECODE_SPLIT
#define HSWA_DECODE_SPLIT 8192
#endif
constexpr int SPLIT = HSWA_DECODE_SPLIT;  // cached keys per split (tuning parameter, multiple of KB)
static_assert(SPLIT % 64 == 0, "splits start on page boundaries");

struct WsHeader {
  int counter;
  int total_items;
  int body_total;  // splits before each sequence's last one, summed over all sequences
  int pad[61];
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace: header, the work-list plan (five int arrays over the sequences), then one
// (m, l, O) partial per work item.
struct WsLayout {
  size_t part_off, part_bytes_per_item, bytes;
  __host__ __device__ WsLayout(int n_seqs, int rows, int d, int64_t max_items) {
    part_off = align256(sizeof(WsHeader) + sizeof(int) * (5 * (size_t)n_seqs + 1));
    part_bytes_per_item = (size_t)rows * (d + 2) * sizeof(float);
    bytes = part_off + part_bytes_per_item * (size_t)max_items;
  }
};

// The order in which the persistent CTAs take work (built by plan_kernel each call).
// Every split of a sequence but its last covers exactly SPLIT cached keys ("body" splits); the
// last one ("tail") holds the rest plus the new tokens. The work list is
//   part A: the body splits, sequence by sequence, longest length bucket first
//           (>= 256K tokens, 64K..256K, < 64K; stable within a bucket);
//   part B: one tail split per sequence, in descending size classes of SPLIT/8 keys.
// Heavy items start first and the step ends on the lightest ones, so the CTAs finish together.
struct PlanView {
  int* prefix;  // [n + 1] body splits before position pos of part A
  int* order;   // [n] part-A position -> sequence
  int* inv_a;   // [n] sequence -> part-A position
  int* tail;    // [n] part-B position -> sequence
  int* inv_b;   // [n] sequence -> part-B position
  __device__ PlanView(uint8_t* ws, int n) {
    prefix = reinterpret_cast<int*>(ws + sizeof(WsHeader));
    order = prefix + n + 1;
    inv_a = order + n;
    tail = inv_a + n;
    inv_b = tail + n;
  }
};

constexpr int NCLS_A = 3;  // length buckets of part A
constexpr int NCLS_B = 8;  // size classes of part B

struct DecParams {
  int n_seqs, n_qt, Hq, Hkv, G, R, window;
  const uint16_t* q;
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t* o;
  const int64_t* ctx_len;
  int64_t max_ctx_len;
  const int32_t* seq_ids;
  const int32_t* page_table;
  int pt_stride;
  const uint16_t* src_k;  // ring or page base of the layer
  const uint16_t* src_v;
  const uint8_t* src_k8;  // the same, as bytes
  const uint8_t* src_v8;
  const float* k_scale;   // FP8 pools: per KV head of this layer: scale and reciprocal of K and V
  const float* v_scale;
  const float* inv_k;
  const float* inv_v;
  int n_swa, ring_layer, max_seqs;
  int full_layer;
  int64_t pages;
  float scale_log2;
  uint8_t* ws;
  size_t part_off, part_bytes;
  int* err;
};

__device__ __forceinline__ int64_t dec_klo(const DecParams& p, int64_t L) {
  if (p.window <= 0) return 0;
  const int64_t lo = L - p.window + 1;
  return lo > 0 ? lo : 0;
}

__device__ __forceinline__ int n_splits(const DecParams& p, int64_t L) {
  const int64_t cached = L - dec_klo(p, L);
  const int64_t n = (cached + SPLIT - 1) / SPLIT;
  return n < 1 ? 1 : (int)n;
}

__device__ __forceinline__ int64_t safe_len(const DecParams& p, int s) {
  int64_t L = p.ctx_len[s];
  if (L < 0 || L > p.max_ctx_len) {
    record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
    L = 0;
  }
  return L;
}

// Length bucket of a sequence (part A order: higher first).
__device__ __forceinline__ int class_a(int64_t L) { return L >= 262144 ? 2 : (L >= 65536 ? 1 : 0); }

// Size class of a sequence's last split (part B order: higher first).
__device__ __forceinline__ int class_b(const DecParams& p, int64_t L) {
  const int64_t cached = L - dec_klo(p, L);
  const int64_t tail = cached - (int64_t)(n_splits(p, L) - 1) * SPLIT;  // 0 .. SPLIT
  const int c = (int)(tail / (SPLIT / NCLS_B));
  return c < NCLS_B - 1 ? c : NCLS_B - 1;
}

// Builds the work list (see PlanView) and resets the work counter. One block of 1024 threads:
// class totals, then a stable placement chunk by chunk (warp ballots give each thread its rank
// among earlier threads of its class), then prefix sums of the body splits in part-A order.
__global__ void __launch_bounds__(1024) plan_kernel(DecParams p) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  PlanView pv(p.ws, p.n_seqs);
  constexpr int NC = NCLS_A + NCLS_B;
  __shared__ int cnt[NC];      // sequences per class (classes 0..2: part A, 3..10: part B)
  __shared__ int cur[NC];      // next position of each class
  __shared__ int wcnt[NC][32]; // this chunk: per-warp counts, then exclusive per-warp offsets
  __shared__ int chunk_tot[NC];
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid < NC) cnt[tid] = 0;
  __syncthreads();
  for (int base = 0; base < p.n_seqs; base += 1024) {
    const int s = base + tid;
    if (s < p.n_seqs) {
      const int64_t L = safe_len(p, s);
      atomicAdd(&cnt[class_a(L)], 1);
      atomicAdd(&cnt[NCLS_A + class_b(p, L)], 1);
    }
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int k = NCLS_A - 1; k >= 0; --k) {
      cur[k] = acc;
      acc += cnt[k];
    }
    acc = 0;
    for (int k = NC - 1; k >= NCLS_A; --k) {
      cur[k] = acc;
      acc += cnt[k];
    }
  }
  __syncthreads();
  const unsigned lanes_below = (1u << lane) - 1u;
  for (int base = 0; base < p.n_seqs; base += 1024) {
    const int s = base + tid;
    const bool live = s < p.n_seqs;
    int ca = -1, cb = -1;
    if (live) {
      const int64_t L = safe_len(p, s);
      ca = class_a(L);
      cb = NCLS_A + class_b(p, L);
    }
    int rank_a = 0, rank_b = 0;
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      const unsigned m = __ballot_sync(0xffffffffu, k < NCLS_A ? ca == k : cb == k);
      if (lane == 0) wcnt[k][w] = __popc(m);
      if (k == ca) rank_a = __popc(m & lanes_below);
      if (k == cb) rank_b = __popc(m & lanes_below);
    }
    __syncthreads();
    if (w < NC) {  // warp k: exclusive scan of class k's per-warp counts
      const int v = wcnt[w][lane];
      int x = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
      }
      wcnt[w][lane] = x - v;
      if (lane == 31) chunk_tot[w] = x;
    }
    __syncthreads();
    if (live) {
      const int pa = cur[ca] + wcnt[ca][w] + rank_a;
      const int pb = cur[cb] + wcnt[cb][w] + rank_b;
      pv.order[pa] = s;
      pv.inv_a[s] = pa;
      pv.tail[pb] = s;
      pv.inv_b[s] = pb;
    }
    __syncthreads();
    if (tid < NC) cur[tid] += chunk_tot[tid];
    __syncthreads();
  }
  // prefix sums of the body splits over part-A positions (block-wide inclusive scan per chunk)
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < p.n_seqs; base += 1024) {
    const int pos = base + tid;
    const int v = pos < p.n_seqs ? n_splits(p, safe_len(p, pv.order[pos])) - 1 : 0;
    int x = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
      int ws_ = warp_sums[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ws_, d);
        if (lane >= d) ws_ += y;
      }
      warp_sums[lane] = ws_;
    }
    __syncthreads();
    const int incl = x + (w > 0 ? warp_sums[w - 1] : 0) + carry;
    if (pos < p.n_seqs) pv.prefix[pos + 1] = incl;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
  if (tid == 0) {
    pv.prefix[0] = 0;
    hdr->body_total = carry;
    hdr->total_items = (carry + p.n_seqs) * p.Hkv;
    hdr->counter = 0;
  }
}

// ---------------------------------------------------------------- mma.sync helpers

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two fp32 -> packed f16x2 (round to nearest even, saturating at +-65504); lo in the low half.
__device__ __forceinline__ uint32_t pack_f16x2_sat(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 codes (low byte, high byte of x's low 16 bits) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t x) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(x));
  return r;
}

// byte offset of 16-byte chunk `c` of row `r` in a [rows][D] bf16 (or f16) tile, XOR-swizzled
template <int D>
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

// byte offset of 16-byte chunk `c` of row `r` in a [rows][D] FP8 tile (rows of D bytes), XOR-swizzled
// so that the 8 rows an ldmatrix reads fall in distinct banks
template <int D>
__device__ __forceinline__ uint32_t sw8_off(int r, int c) {
  if constexpr (D == 128) return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
  else return (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

template <int D, int MT, bool FP8>
struct DecSmem {
  static constexpr int ROWS = 16 * MT;
  static constexpr int NS = FP8 ? NST8 : NST;      // pipeline stages
  static constexpr int TILE = KB * D * (FP8 ? 1 : 2);
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + NS * TILE;
  static constexpr int Q_OFF = V_OFF + NS * TILE;  // Q rows, bf16 (or f16 with FP8 blocks)
  static constexpr int MISC_OFF = Q_OFF + ROWS * D * 2;
  // merge area aliases the K/V stages (idle while merging)
  static constexpr int ACC_OFF = 0;
  static constexpr int BYTES = MISC_OFF + 4 * ROWS * 4 * 2 + ROWS * 4 * 2 + 64;
  static_assert(4 * ROWS * (D + 8) * 4 <= 2 * NS * TILE, "merge regions must fit in the K/V stages");
};

// FP8 blocks (pools of E4M3 codes): the block copies move half the bytes; S = Q K^T and O += P V
// run on f16 MMAs (E4M3 -> f16 is exact) with Q and P in f16, fragments built straight from the
// FP8 bytes in shared memory:
//  * K: ldmatrix of an 8-key x 16-byte FP8 matrix gives each thread 4 consecutive dims of one key,
//    i.e. B-fragment k slots (2l, 2l+1, 2l+8, 2l+9) hold dims (4l, 4l+1, 4l+2, 4l+3); Q is staged
//    with its dims permuted the same way in each 16-dim group, so every dot product is unchanged.
//  * V: ldmatrix.trans of the same matrix gives each thread two keys x two adjacent dims; its even
//    and odd dims form the B fragments of two n-tiles ("even" n-tile 2c holds dims 16c + 2j,
//    "odd" n-tile 2c + 1 dims 16c + 2j + 1), put back in order when O leaves the registers.
//  * The K scale of the KV head multiplies the softmax scale; the V scale multiplies O. The new
//    tokens are quantized with the layer's reciprocal scales as they are staged, the values the
//    cache holds once they are committed.
template <int D, int MT, bool FP8>
__global__ void __launch_bounds__(DEC_THREADS, 2) decode_kernel(DecParams p) {
  using SM = DecSmem<D, MT, FP8>;
  constexpr int ROWS = SM::ROWS;
  constexpr int NS = SM::NS;
  constexpr int CH = FP8 ? D / 16 : D / 8;  // 16-byte chunks per K/V row
  extern __shared__ __align__(128) uint8_t smem[];
  float* m_w = reinterpret_cast<float*>(smem + SM::MISC_OFF);   // [4][ROWS]
  float* l_w = m_w + 4 * ROWS;                                  // [4][ROWS]
  float* m_all = l_w + 4 * ROWS;                                // [ROWS]
  float* l_all = m_all + ROWS;                                  // [ROWS]
  int* item_slot = reinterpret_cast<int*>(l_all + ROWS);
  const uint32_t s_base = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  const PlanView pv(p.ws, p.n_seqs);

  if (read_error(p.err) != 0) return;

  // this thread's fixed place in a 64-row block copy: row (within a pass), 16-byte chunk
  const int cp_row = tid / CH;                  // 0 .. 128/CH - 1
  const int cp_chunk = tid % CH;
  constexpr int CP_ROWS = DEC_THREADS / CH;     // rows covered by the CTA per copy instruction
  static_assert(KB % CP_ROWS == 0, "block rows");

  for (;;) {
    if (tid == 0) *item_slot = atomicAdd(&hdr->counter, 1);
    __syncthreads();
    const int item = *item_slot;
    __syncthreads();
    if (item >= hdr->total_items) break;
    const int g = item % p.Hkv;
    const int sc = item / p.Hkv;
    int s, c;
    if (sc < hdr->body_total) {
      // part A: the position pos with prefix[pos] <= sc < prefix[pos + 1] (the largest such pos
      // skips positions without body splits)
      int lo = 0, hi = p.n_seqs;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pv.prefix[mid] <= sc) lo = mid; else hi = mid;
      }
      s = pv.order[lo];
      c = sc - pv.prefix[lo];
    } else {
      s = pv.tail[sc - hdr->body_total];  // part B: the sequence's last split
      c = -1;
    }
    const int L = (int)safe_len(p, s);
    const int nsp = n_splits(p, L);
    if (c < 0) c = nsp - 1;
    const bool last = c == nsp - 1;
    const int klo = (int)dec_klo(p, L);
    const int a = klo + c * SPLIT;
    const int b = (a + SPLIT < L) ? a + SPLIT : L;
    const int n_cached_blk = (b - a + KB - 1) / KB;
    const int n_blk = n_cached_blk + (last ? 1 : 0);
    // source rows of this (sequence, KV head), as bytes
    constexpr int RB = FP8 ? D : 2 * D;  // bytes per K/V row
    const uint8_t* ring_k = nullptr;
    const uint8_t* ring_v = nullptr;
    bool src_ok = true;
    if (p.window > 0) {
      const int seq = p.seq_ids[s];
      if (seq < 0 || seq >= p.max_seqs) {
        record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
        src_ok = false;
      } else {
        const int64_t row0 = (((int64_t)seq * p.n_swa + p.ring_layer) * p.Hkv + g) * p.window;
        ring_k = p.src_k8 + row0 * RB;
        ring_v = p.src_v8 + row0 * RB;
      }
    }
    const int32_t* pt_row = p.page_table ? p.page_table + (int64_t)s * p.pt_stride : nullptr;

    // ---- block loader: block kb2 of this item into stage st. Each copy instruction of the CTA
    // moves CP_ROWS whole rows (contiguous in HBM within a page or a ring run).
    auto kv_off = [](int r, int c) -> uint32_t {
      if constexpr (FP8) return sw8_off<D>(r, c);
      else return sw_off<D>(r, c);
    };
    auto load_block = [&](int kb2, int st) {
      const uint32_t kdst = s_base + SM::K_OFF + st * SM::TILE;
      const uint32_t vdst = s_base + SM::V_OFF + st * SM::TILE;
      if (kb2 < n_cached_blk) {
        const int pos0 = a + kb2 * KB;
        const int nvalid = b - pos0;  // rows of this block that exist (>= 1)
        if (p.window > 0) {
          int slot0 = pos0 % p.window;
#pragma unroll
          for (int rr = 0; rr < KB; rr += CP_ROWS) {
            const int r = rr + cp_row;
            int slot = slot0 + r;
            if (slot >= p.window) slot = (p.window >= KB) ? slot - p.window : slot % p.window;
            const bool ok = src_ok && r < nvalid;
            const size_t off = ok ? (size_t)slot * RB + cp_chunk * 16 : 0;
            const uint8_t* sk = ok ? ring_k + off : p.src_k8;
            const uint8_t* sv = ok ? ring_v + off : p.src_v8;
            cp_async_16(kdst + kv_off(r, cp_chunk), sk, ok ? 16u : 0u);
            cp_async_16(vdst + kv_off(r, cp_chunk), sv, ok ? 16u : 0u);
          }
        } else {
          // a block is exactly one 64-token page (splits start at multiples of 64)
          const int lp = pos0 / 64;
          int32_t page = lp < p.pt_stride ? pt_row[lp] : -1;
          bool ok_page = page >= 0 && page < p.pages;
          if (!ok_page && tid == 0) record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
          const int64_t prow = ok_page ? (((int64_t)p.full_layer * p.pages + page) * p.Hkv + g) * 64 : 0;
          const uint8_t* kbase = p.src_k8 + prow * RB;
          const uint8_t* vbase = p.src_v8 + prow * RB;
#pragma unroll
          for (int rr = 0; rr < KB; rr += CP_ROWS) {
            const int r = rr + cp_row;
            const bool ok = ok_page && r < nvalid;
            const int off = ok ? r * RB + cp_chunk * 16 : 0;
            cp_async_16(kdst + kv_off(r, cp_chunk), ok ? kbase + off : p.src_k8, ok ? 16u : 0u);
            cp_async_16(vdst + kv_off(r, cp_chunk), ok ? vbase + off : p.src_v8, ok ? 16u : 0u);
          }
        }
      } else if constexpr (FP8) {
        // the new tokens, quantized as the cache will hold them: rows 0 .. n_qt-1, zeros after
        const float ik = p.inv_k[g], iv = p.inv_v[g];
        auto q16 = [](const uint16_t* src, float inv) -> uint4 {
          const uint4 x0 = reinterpret_cast<const uint4*>(src)[0], x1 = reinterpret_cast<const uint4*>(src)[1];
          const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t lo = pack_e4m3x2(__uint_as_float(w[2 * i] << 16) * inv,
                                            __uint_as_float(w[2 * i] & 0xFFFF0000u) * inv);
            const uint32_t hi = pack_e4m3x2(__uint_as_float(w[2 * i + 1] << 16) * inv,
                                            __uint_as_float(w[2 * i + 1] & 0xFFFF0000u) * inv);
            o[i] = lo | (hi << 16);
          }
          return make_uint4(o[0], o[1], o[2], o[3]);
        };
#pragma unroll
        for (int rr = 0; rr < KB; rr += CP_ROWS) {
          const int r = rr + cp_row;
          uint4 qk = make_uint4(0, 0, 0, 0), qv = make_uint4(0, 0, 0, 0);
          if (r < p.n_qt) {
            const int64_t row = ((int64_t)s * p.n_qt + r) * p.Hkv + g;
            qk = q16(p.k_new + row * D + cp_chunk * 16, ik);
            qv = q16(p.v_new + row * D + cp_chunk * 16, iv);
          }
          *reinterpret_cast<uint4*>(smem + SM::K_OFF + st * SM::TILE + kv_off(r, cp_chunk)) = qk;
          *reinterpret_cast<uint4*>(smem + SM::V_OFF + st * SM::TILE + kv_off(r, cp_chunk)) = qv;
        }
      } else {
        // the new tokens: rows 0 .. n_qt-1 of k_new / v_new, zeros after
#pragma unroll
        for (int rr = 0; rr < KB; rr += CP_ROWS) {
          const int r = rr + cp_row;
          const bool ok = r < p.n_qt;
          const int64_t row = ((int64_t)s * p.n_qt + (ok ? r : 0)) * p.Hkv + g;
          const uint16_t* sk = p.k_new + row * D + cp_chunk * 8;
          const uint16_t* sv = p.v_new + row * D + cp_chunk * 8;
          cp_async_16(kdst + kv_off(r, cp_chunk), sk, ok ? 16u : 0u);
          cp_async_16(vdst + kv_off(r, cp_chunk), sv, ok ? 16u : 0u);
        }
      }
    };

#pragma unroll
    for (int st = 0; st < NS - 1; ++st) {
      if (st < n_blk) load_block(st, st);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }

    // Q is staged while the first blocks' copies are in flight (the block loop's first barrier
    // orders it before its first use)
    // ---- stage Q rows (row = t * G + hh) into shared memory, zero rows >= R
    if constexpr (FP8) {
      // f16, dims of each 16-dim group in the order (0,1,4,5,8,9,12,13 | 2,3,6,7,10,11,14,15)
      for (int idx = tid; idx < ROWS * (D / 16); idx += DEC_THREADS) {
        const int r = idx / (D / 16), grp = idx % (D / 16);
        uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (r < p.R) {
          const int t = r / p.G, hh = r % p.G;
          const uint4* src = reinterpret_cast<const uint4*>(
              p.q + (((int64_t)s * p.n_qt + t) * p.Hq + g * p.G + hh) * D + grp * 16);
          const uint4 x0 = src[0], x1 = src[1];
          w[0] = x0.x; w[1] = x0.y; w[2] = x0.z; w[3] = x0.w;
          w[4] = x1.x; w[5] = x1.y; w[6] = x1.z; w[7] = x1.w;
        }
        // w[i] holds dims 2i (low half) and 2i + 1 (high half) as bf16
        uint32_t c0[4], c1[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // dims 4j, 4j+1 -> chunk 0 slot j; dims 4j+2, 4j+3 -> chunk 1 slot j
          c0[j] = pack_f16x2_sat(__uint_as_float(w[2 * j] << 16), __uint_as_float(w[2 * j] & 0xFFFF0000u));
          c1[j] = pack_f16x2_sat(__uint_as_float(w[2 * j + 1] << 16), __uint_as_float(w[2 * j + 1] & 0xFFFF0000u));
        }
        *reinterpret_cast<uint4*>(smem + SM::Q_OFF + sw_off<D>(r, 2 * grp)) = make_uint4(c0[0], c0[1], c0[2], c0[3]);
        *reinterpret_cast<uint4*>(smem + SM::Q_OFF + sw_off<D>(r, 2 * grp + 1)) =
            make_uint4(c1[0], c1[1], c1[2], c1[3]);
      }
    } else {
      for (int idx = tid; idx < ROWS * (D / 8); idx += DEC_THREADS) {
        const int r = idx / (D / 8), ch = idx % (D / 8);
        uint4 val = make_uint4(0, 0, 0, 0);
        if (r < p.R) {
          const int t = r / p.G, hh = r % p.G;
          const uint16_t* src = p.q + (((int64_t)s * p.n_qt + t) * p.Hq + g * p.G + hh) * D + ch * 8;
          val = *reinterpret_cast<const uint4*>(src);
        }
        *reinterpret_cast<uint4*>(smem + SM::Q_OFF + sw_off<D>(r, ch)) = val;
      }
    }


    // per-thread row state: rows (mt*16 + lane/4) and (+8)
    float o_acc[MT][D / 8][4];
    float m_r[MT][2], l_r[MT][2];
    int row_pos[MT][2], row_lo[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        m_r[mt][hf] = -INFINITY;
        l_r[mt][hf] = 0.f;
        const int r = mt * 16 + (lane >> 2) + hf * 8;
        const int t = r < p.R ? r / p.G : 0;
        row_pos[mt][hf] = L + t;
        int lo2 = 0;
        if (p.window > 0) {
          lo2 = L + t - p.window + 1;
          if (lo2 < 0) lo2 = 0;
        }
        row_lo[mt][hf] = r < p.R ? lo2 : 0x7fffffff;  // padding rows see nothing
      }
#pragma unroll
      for (int nd = 0; nd < D / 8; ++nd) o_acc[mt][nd][0] = o_acc[mt][nd][1] = o_acc[mt][nd][2] = o_acc[mt][nd][3] = 0.f;
    }
    // largest window start over the real rows: cached keys at or above it need no mask
    const int lo_max = p.window > 0 ? (L + p.n_qt - 1 - p.window + 1 > 0 ? L + p.n_qt - p.window : 0) : 0;

    const float sl2 = FP8 ? p.scale_log2 * p.k_scale[g] : p.scale_log2;
    for (int kb2 = 0; kb2 < n_blk; ++kb2) {
      asm volatile("cp.async.wait_group %0;" ::"n"(NS - 2) : "memory");
      __syncthreads();  // block kb2 is visible; every warp is done with block kb2 - 1
      {
        const int nxt = kb2 + NS - 1;
        if (nxt < n_blk) load_block(nxt, nxt % NS);
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      const int st = kb2 % NS;
      const uint32_t kt = s_base + SM::K_OFF + st * SM::TILE;
      const uint32_t vt = s_base + SM::V_OFF + st * SM::TILE;
      const uint32_t qt = s_base + SM::Q_OFF;
      const int key0 = warp * 16;  // this warp's 16 keys of the block

      // S = Q K^T for ROWS x 16 keys
      float sacc[MT][2][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) sacc[mt][nt][0] = sacc[mt][nt][1] = sacc[mt][nt][2] = sacc[mt][nt][3] = 0.f;
      if constexpr (FP8) {
#pragma unroll
        for (int kk = 0; kk < D / 16; kk += 2) {
          // matrices: keys 0-7 / 8-15 of this warp's slice x dims of groups kk and kk + 1
          uint32_t r0, r1, r2, r3;
          {
            const int mi = lane >> 3;
            const int key = key0 + (mi & 1) * 8 + (lane & 7);
            ldsm_x4(kt + sw8_off<D>(key, kk + (mi >> 1)), r0, r1, r2, r3);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t k0 = h ? r2 : r0, k1 = h ? r3 : r1;
            const uint32_t b00 = e4m3x2_to_f16x2(k0), b01 = e4m3x2_to_f16x2(k0 >> 16);
            const uint32_t b10 = e4m3x2_to_f16x2(k1), b11 = e4m3x2_to_f16x2(k1 >> 16);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              uint32_t a0, a1, a2, a3;
              const int mi = lane >> 3;
              const int row = mt * 16 + (mi & 1) * 8 + (lane & 7);
              ldsm_x4(qt + sw_off<D>(row, (kk + h) * 2 + (mi >> 1)), a0, a1, a2, a3);
              mma_f16(sacc[mt][0], a0, a1, a2, a3, b00, b01);
              mma_f16(sacc[mt][1], a0, a1, a2, a3, b10, b11);
            }
          }
        }
      } else {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t b0, b1, b2, b3;
          {
            const int mi = lane >> 3;
            const int key = key0 + (mi >> 1) * 8 + (lane & 7);
            ldsm_x4(kt + sw_off<D>(key, kk * 2 + (mi & 1)), b0, b1, b2, b3);
          }
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            uint32_t a0, a1, a2, a3;
            const int mi = lane >> 3;
            const int row = mt * 16 + (mi & 1) * 8 + (lane & 7);
            ldsm_x4(qt + sw_off<D>(row, kk * 2 + (mi >> 1)), a0, a1, a2, a3);
            mma_bf16(sacc[mt][0], a0, a1, a2, a3, b0, b1);
            mma_bf16(sacc[mt][1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
      // mask (edge blocks only) + online softmax in the exp2 domain with lazy rescaling
      const bool is_new = kb2 >= n_cached_blk;
      const int kpos_base = is_new ? L : a + kb2 * KB;
      const bool need_mask = is_new || kpos_base + KB > b || kpos_base < lo_max;
      uint32_t pa[MT][4];
      // this lane's key columns are key0 + (lane & 3) * 2 + {0, 1, 8, 9}
      const int col_base = kpos_base + key0 + (lane & 3) * 2;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          // FP8 blocks: raw scores, the scale (> 0) applied to the row maximum and inside the
          // exponential's FMA (max(s) * c = max(s * c) exactly, rounding being monotone; measured 2%
          // faster there); bf16 blocks: scaled scores (the other form measured 1.6% slower there)
          float v[4];
          if constexpr (FP8) {
            v[0] = sacc[mt][0][hf * 2 + 0];
            v[1] = sacc[mt][0][hf * 2 + 1];
            v[2] = sacc[mt][1][hf * 2 + 0];
            v[3] = sacc[mt][1][hf * 2 + 1];
            if (need_mask) {
              // allowed offsets j (key = col_base + j) for this row: lo_j <= j < hi_j
              const int hi_pos = is_new ? min(L + p.n_qt, row_pos[mt][hf] + 1) : b;  // exclusive
              const int lo_j = row_lo[mt][hf] - col_base;
              const int hi_j = hi_pos - col_base;
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                const int j = (x >> 1) * 8 + (x & 1);
                if (!(j >= lo_j && j < hi_j)) v[x] = -INFINITY;
              }
            }
          } else {
            // allowed offsets j (key = col_base + j) for this row: lo_j <= j < hi_j
            int lo_j = 0, hi_j = 16;
            if (need_mask) {
              const int hi_pos = is_new ? min(L + p.n_qt, row_pos[mt][hf] + 1) : b;  // exclusive
              lo_j = row_lo[mt][hf] - col_base;
              hi_j = hi_pos - col_base;
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int j = nt * 8 + e;
                const float sv = sacc[mt][nt][hf * 2 + e] * sl2;
                v[nt * 2 + e] = (j >= lo_j && j < hi_j) ? sv : -INFINITY;
              }
          }
          float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          if constexpr (FP8) mx *= sl2;
          // lazy rescale: move the offset only when the maximum grew by more than 2^8
          if (mx > m_r[mt][hf] + 8.f) {
            const float alpha = ex2_approx(m_r[mt][hf] - mx);  // 0 when the old offset is -inf
            m_r[mt][hf] = mx;
            l_r[mt][hf] *= alpha;
#pragma unroll
            for (int nd = 0; nd < D / 8; ++nd) {
              o_acc[mt][nd][hf * 2 + 0] *= alpha;
              o_acc[mt][nd][hf * 2 + 1] *= alpha;
            }
          }
          const float moff = m_r[mt][hf] == -INFINITY ? 0.f : m_r[mt][hf];
          float pv[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) pv[x] = FP8 ? ex2_approx(fmaf(v[x], sl2, -moff)) : ex2_approx(v[x] - moff);
          l_r[mt][hf] += (pv[0] + pv[1]) + (pv[2] + pv[3]);
          // A fragment of P (16 rows x 16 keys): a0/a1 = keys 0-7 (rows r, r+8), a2/a3 = keys 8-15
          if constexpr (FP8) {
            pa[mt][hf + 0] = pack_f16x2_sat(pv[0], pv[1]);
            pa[mt][hf + 2] = pack_f16x2_sat(pv[2], pv[3]);
          } else {
            pa[mt][hf + 0] = pack_bf16x2(pv[0], pv[1]);
            pa[mt][hf + 2] = pack_bf16x2(pv[2], pv[3]);
          }
        }
      }
      // O += P V  (16 keys x D)
      if constexpr (FP8) {
#pragma unroll
        for (int c2 = 0; c2 < D / 16; c2 += 2) {
          // matrices: keys 0-7 / 8-15 of this warp's slice x the 16 dims of groups c2 and c2 + 1;
          // transposed, each register holds keys (2l, 2l + 1) x dims (2j, 2j + 1), j = lane / 4
          uint32_t r0, r1, r2, r3;
          {
            const int mi = lane >> 3;
            const int key = key0 + (mi & 1) * 8 + (lane & 7);
            ldsm_x4_t(vt + sw8_off<D>(key, c2 + (mi >> 1)), r0, r1, r2, r3);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t v0 = h ? r2 : r0, v1 = h ? r3 : r1;
            // even dims: bytes 0 and 2 (keys 2l, 2l + 1 of dim 2j); odd dims: bytes 1 and 3
            const uint32_t be0 = e4m3x2_to_f16x2(__byte_perm(v0, 0u, 0x0020u));
            const uint32_t be1 = e4m3x2_to_f16x2(__byte_perm(v1, 0u, 0x0020u));
            const uint32_t bo0 = e4m3x2_to_f16x2(__byte_perm(v0, 0u, 0x0031u));
            const uint32_t bo1 = e4m3x2_to_f16x2(__byte_perm(v1, 0u, 0x0031u));
            const int grp = c2 + h;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              mma_f16(o_acc[mt][2 * grp + 0], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], be0, be1);
              mma_f16(o_acc[mt][2 * grp + 1], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], bo0, bo1);
            }
          }
        }
      } else {
#pragma unroll
        for (int nd2 = 0; nd2 < D / 16; ++nd2) {
          uint32_t b0, b1, b2, b3;
          const int mi = lane >> 3;
          const int key = key0 + (mi & 1) * 8 + (lane & 7);
          ldsm_x4_t(vt + sw_off<D>(key, nd2 * 2 + (mi >> 1)), b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            mma_bf16(o_acc[mt][nd2 * 2 + 0], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], b0, b1);
            mma_bf16(o_acc[mt][nd2 * 2 + 1], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], b2, b3);
          }
        }
      }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");

    // ---- merge the 4 warps' states
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float lsum = l_r[mt][hf];
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
        l_r[mt][hf] = lsum;
        if ((lane & 3) == 0) {
          const int r = mt * 16 + (lane >> 2) + hf * 8;
          m_w[warp * ROWS + r] = m_r[mt][hf];
          l_w[warp * ROWS + r] = lsum;
        }
      }
    // each warp's partial O, rescaled to the rows' common maximum, goes to its own region of the
    // (now idle) K/V stage buffers; the output pass sums the four regions (no shared atomics)
    constexpr int RS = D + 8;  // padded row stride: a warp's float2 stores hit distinct banks
    float* part_w = reinterpret_cast<float*>(smem + SM::ACC_OFF);  // [4][ROWS][RS]
    static_assert(4 * ROWS * RS * 4 <= 2 * NS * SM::TILE, "merge regions must fit in the K/V stages");
    __syncthreads();
    for (int r = tid; r < ROWS; r += DEC_THREADS) {
      float M = -INFINITY;
      for (int w = 0; w < 4; ++w) M = fmaxf(M, m_w[w * ROWS + r]);
      const float Mo = M == -INFINITY ? 0.f : M;
      float Ls = 0.f;
      for (int w = 0; w < 4; ++w) Ls += l_w[w * ROWS + r] * ex2_approx(m_w[w * ROWS + r] - Mo);
      m_all[r] = M;
      l_all[r] = Ls;
    }
    __syncthreads();
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = mt * 16 + (lane >> 2) + hf * 8;
        const float Mo = m_all[r] == -INFINITY ? 0.f : m_all[r];
        const float f = ex2_approx(m_r[mt][hf] - Mo);
        if constexpr (FP8) {
          // n-tiles 2c (even dims) and 2c + 1 (odd dims) of group c: this thread's dims 16c + 4l .. + 3
          float* dst = part_w + (warp * ROWS + r) * RS + (lane & 3) * 4;
#pragma unroll
          for (int c = 0; c < D / 16; ++c)
            *reinterpret_cast<float4*>(dst + c * 16) =
                make_float4(o_acc[mt][2 * c][hf * 2 + 0] * f, o_acc[mt][2 * c + 1][hf * 2 + 0] * f,
                            o_acc[mt][2 * c][hf * 2 + 1] * f, o_acc[mt][2 * c + 1][hf * 2 + 1] * f);
        } else {
          float* dst = part_w + (warp * ROWS + r) * RS + (lane & 3) * 2;
#pragma unroll
          for (int nd = 0; nd < D / 8; ++nd)
            *reinterpret_cast<float2*>(dst + nd * 8) =
                make_float2(o_acc[mt][nd][hf * 2 + 0] * f, o_acc[mt][nd][hf * 2 + 1] * f);
        }
      }
    __syncthreads();
    // element (r, c) of the merged, unnormalised O
    auto merged4 = [&](int r, int c) -> float4 {
      float4 x = *reinterpret_cast<const float4*>(part_w + (0 * ROWS + r) * RS + c);
#pragma unroll
      for (int w = 1; w < 4; ++w) {
        const float4 y = *reinterpret_cast<const float4*>(part_w + (w * ROWS + r) * RS + c);
        x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
      }
      return x;
    };
    __syncthreads();
    const float vs = FP8 ? p.v_scale[g] : 1.f;  // the V scale of an FP8 pool multiplies O
    if (nsp == 1) {
      // single split: normalise and write bf16 output rows
      for (int idx = tid; idx < p.R * (D / 8); idx += DEC_THREADS) {
        const int r = idx / (D / 8), ch = idx % (D / 8);
        const float inv = vs / l_all[r];
        const float4 lo4 = merged4(r, ch * 8), hi4 = merged4(r, ch * 8 + 4);
        uint4 pk;
        pk.x = pack_bf16x2(lo4.x * inv, lo4.y * inv);
        pk.y = pack_bf16x2(lo4.z * inv, lo4.w * inv);
        pk.z = pack_bf16x2(hi4.x * inv, hi4.y * inv);
        pk.w = pack_bf16x2(hi4.z * inv, hi4.w * inv);
        const int t = r / p.G, hh = r % p.G;
        uint16_t* dst = p.o + (((int64_t)s * p.n_qt + t) * p.Hq + g * p.G + hh) * D + ch * 8;
        *reinterpret_cast<uint4*>(dst) = pk;
      }
    } else {
      float* part = reinterpret_cast<float*>(p.ws + p.part_off + (size_t)item * p.part_bytes);
      for (int idx = tid; idx < p.R * (D / 4); idx += DEC_THREADS) {
        const int r = idx / (D / 4), c = (idx % (D / 4)) * 4;
        float4 x = merged4(r, c);
        if constexpr (FP8) {
          x.x *= vs; x.y *= vs; x.z *= vs; x.w *= vs;
        }
        *reinterpret_cast<float4*>(part + r * D + c) = x;
      }
      for (int r = tid; r < p.R; r += DEC_THREADS) {
        part[p.R * D + r] = m_all[r];
        part[p.R * D + p.R + r] = l_all[r];
      }
    }
    __syncthreads();
  }
}

// One CTA of 256 threads per (sequence, KV head) with more than one split.
//  phase 1: 8 threads per row reduce the splits' maxima M and denominators sum_c 2^(m_c - M) l_c
//           (shuffles within the 8-thread group), keeping the factors 2^(m_c - M) in shared memory;
//  phase 2: each thread owns 4 float4 groups of the R x D output and walks the splits with
//           8 independent loads in flight.
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(DecParams p) {
  const int g = blockIdx.x % p.Hkv;
  const int s = blockIdx.x / p.Hkv;
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(p.ws);
  const PlanView pv(p.ws, p.n_seqs);
  const int nsp = n_splits(p, safe_len(p, s));
  if (nsp <= 1) return;
  extern __shared__ float msh[];  // [nsp][R] scale factors, then [R] inverse denominators
  float* fac = msh;
  float* inv = msh + (size_t)nsp * p.R;
  // partials of this (s, g): body splits are consecutive items of part A, the last split is in part B
  const uint8_t* body0 = p.ws + p.part_off + ((size_t)pv.prefix[pv.inv_a[s]] * p.Hkv + g) * p.part_bytes;
  const uint8_t* tailp = p.ws + p.part_off + ((size_t)(hdr->body_total + pv.inv_b[s]) * p.Hkv + g) * p.part_bytes;
  const size_t split_stride = (size_t)p.Hkv * p.part_bytes;
  auto split_part = [&](int c) -> const float* {
    return reinterpret_cast<const float*>(c < nsp - 1 ? body0 + (size_t)c * split_stride : tailp);
  };
  const int lane8 = threadIdx.x & 7;
  // rows padded to whole warps (4 rows of 8 threads per warp) so every shuffle has all 32 lanes
  const int r_pad = (p.R + 3) & ~3;
  for (int r = threadIdx.x >> 3; r < r_pad; r += 32) {
    const bool live = r < p.R;
    float M = -INFINITY;
    for (int c = lane8; live && c < nsp; c += 8)
      M = fmaxf(M, split_part(c)[p.R * D + r]);
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 1));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 4));
    const float Mo = M == -INFINITY ? 0.f : M;
    float den = 0.f;
    for (int c = lane8; live && c < nsp; c += 8) {
      const float* part = split_part(c);
      const float f = ex2_approx(part[p.R * D + r] - Mo);
      fac[c * p.R + r] = f;
      den += f * part[p.R * D + p.R + r];
    }
    den += __shfl_xor_sync(0xffffffffu, den, 1);
    den += __shfl_xor_sync(0xffffffffu, den, 2);
    den += __shfl_xor_sync(0xffffffffu, den, 4);
    if (live && lane8 == 0) inv[r] = 1.f / den;
  }
  __syncthreads();
  constexpr int Q4 = D / 4;  // float4 groups per row
  const int n_items = p.R * Q4;
  for (int base = threadIdx.x; base < n_items; base += 4 * blockDim.x) {
    float4 acc[4];
    int it_r[4], it_c[4];
    bool ok[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * blockDim.x;
      ok[u] = idx < n_items;
      it_r[u] = ok[u] ? idx / Q4 : 0;
      it_c[u] = ok[u] ? (idx % Q4) * 4 : 0;
      acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    int c = 0;
    for (; c + 2 <= nsp; c += 2) {
      const float* pa = split_part(c);
      const float* pb = split_part(c + 1);
      float4 va[4], vb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        va[u] = *reinterpret_cast<const float4*>(pa + it_r[u] * D + it_c[u]);
        vb[u] = *reinterpret_cast<const float4*>(pb + it_r[u] * D + it_c[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float fa = fac[c * p.R + it_r[u]], fb = fac[(c + 1) * p.R + it_r[u]];
        acc[u].x += fa * va[u].x + fb * vb[u].x;
        acc[u].y += fa * va[u].y + fb * vb[u].y;
        acc[u].z += fa * va[u].z + fb * vb[u].z;
        acc[u].w += fa * va[u].w + fb * vb[u].w;
      }
    }
    if (c < nsp) {
      const float* pa = split_part(c);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 va = *reinterpret_cast<const float4*>(pa + it_r[u] * D + it_c[u]);
        const float fa = fac[c * p.R + it_r[u]];
        acc[u].x += fa * va.x;
        acc[u].y += fa * va.y;
        acc[u].z += fa * va.z;
        acc[u].w += fa * va.w;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (!ok[u]) continue;
      const int r = it_r[u];
      const float iv = inv[r];
      const int t = r / p.G, hh = r % p.G;
      uint16_t* dst = p.o + (((int64_t)s * p.n_qt + t) * p.Hq + g * p.G + hh) * D + it_c[u];
      uint2 pk;
      pk.x = pack_bf16x2(acc[u].x * iv, acc[u].y * iv);
      pk.y = pack_bf16x2(acc[u].z * iv, acc[u].w * iv);
      *reinterpret_cast<uint2*>(dst) = pk;
    }
  }
}

#include "decode_tc.cuh"

// Largest split count of any sequence for these arguments.
int64_t max_splits(int window, int64_t max_ctx_len) {
  const int64_t cached = window > 0 ? (max_ctx_len < window ? max_ctx_len : window - 1) : max_ctx_len;
  const int64_t nsp = (cached + SPLIT - 1) / SPLIT;
  return nsp < 1 ? 1 : nsp;
}

template <int D, int MT, bool FP8>
int launch_t(DecParams& p, int n_items_max, int sms, size_t merge_smem, cudaStream_t stream) {
  using SM = DecSmem<D, MT, FP8>;
  plan_kernel<<<1, 1024, 0, stream>>>(p);
  cudaFuncSetAttribute(decode_kernel<D, MT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::BYTES);
  int per_sm = 2;
  int grid = sms * per_sm;
  if (grid > n_items_max) grid = n_items_max;
  if (grid < 1) grid = 1;
  decode_kernel<D, MT, FP8><<<grid, DEC_THREADS, SM::BYTES, stream>>>(p);
  if (merge_smem > 0) {
    if (merge_smem > 48 * 1024)
      cudaFuncSetAttribute(merge_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)merge_smem);
    merge_kernel<D><<<p.n_seqs * p.Hkv, 256, merge_smem, stream>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("hybrid_decode_fwd: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

int launch_tc(DecParams& p, int n_items_max, int sms, size_t merge_smem, cudaStream_t stream) {
  plan_kernel<<<1, 1024, 0, stream>>>(p);
  const int smem = TcLayout::BYTES + 1024;
  cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  int grid = sms < n_items_max ? sms : n_items_max;
  if (grid < 1) grid = 1;
  decode_tc_kernel<<<grid, TC_THREADS, smem, stream>>>(p);
  if (merge_smem > 0) {
    if (merge_smem > 48 * 1024)
      cudaFuncSetAttribute(merge_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)merge_smem);
    merge_kernel<128><<<p.n_seqs * p.Hkv, 256, merge_smem, stream>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("hybrid_decode_fwd: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

}  // namespace

size_t decode_workspace_bytes(int n_seqs, int n_qt, int Hq, int Hkv, int d, int window, int64_t max_ctx_len) {
  const int G = Hq / Hkv;
  const int rows = n_qt * G;
  WsLayout L(n_seqs, rows, d, (int64_t)n_seqs * Hkv * max_splits(window, max_ctx_len));
  return L.bytes;
}

size_t decode_merge_smem_bytes(int n_seqs, int n_qt, int Hq, int Hkv, int window, int64_t max_ctx_len) {
  (void)n_seqs;
  const int64_t nsp = max_splits(window, max_ctx_len);
  if (nsp <= 1) return 0;
  // [nsp][R] scale factors and [R] inverse denominators
  return (size_t)(nsp + 1) * (size_t)(n_qt * (Hq / Hkv)) * sizeof(float);
}

int launch_decode(const DecodeLaunch& Lc, cudaStream_t stream) {
  const hswa_pool* pool = Lc.pool;
  const hswa_pool_desc& D = pool->desc;
  DecParams p{};
  p.n_seqs = Lc.n_seqs;
  p.n_qt = Lc.n_qt;
  p.Hq = Lc.Hq;
  p.Hkv = Lc.Hkv;
  p.G = Lc.Hq / Lc.Hkv;
  p.R = p.n_qt * p.G;
  p.window = Lc.window;
  p.q = Lc.q;
  p.k_new = Lc.k_new;
  p.v_new = Lc.v_new;
  p.o = Lc.o;
  p.ctx_len = Lc.ctx_len;
  p.max_ctx_len = Lc.max_ctx_len;
  p.seq_ids = Lc.seq_ids;
  p.page_table = Lc.page_table;
  p.pt_stride = Lc.pt_stride;
  p.src_k = Lc.window > 0 ? pool->ring_k : pool->page_k;
  p.src_v = Lc.window > 0 ? pool->ring_v : pool->page_v;
  p.src_k8 = Lc.window > 0 ? pool->ring_k8 : pool->page_k8;
  p.src_v8 = Lc.window > 0 ? pool->ring_v8 : pool->page_v8;
  if (pool->fp8) {
    const int n_layers = D.n_swa_layers + D.n_full_layers;
    p.k_scale = pool->scales + (size_t)(0 * n_layers + Lc.layer) * D.n_kv_heads;
    p.v_scale = pool->scales + (size_t)(1 * n_layers + Lc.layer) * D.n_kv_heads;
    p.inv_k = pool->scales + (size_t)(2 * n_layers + Lc.layer) * D.n_kv_heads;
    p.inv_v = pool->scales + (size_t)(3 * n_layers + Lc.layer) * D.n_kv_heads;
  }
  p.n_swa = D.n_swa_layers;
  p.ring_layer = Lc.ring_layer;
  p.max_seqs = D.max_seqs;
  p.full_layer = Lc.full_layer;
  p.pages = D.pages_per_full_layer;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)Lc.d));
  p.ws = static_cast<uint8_t*>(Lc.workspace);
  p.err = pool->err;
  const int64_t mi = (int64_t)p.n_seqs * p.Hkv * max_splits(p.window, p.max_ctx_len);
  WsLayout WL(p.n_seqs, p.R, Lc.d, mi);
  p.part_off = WL.part_off;
  p.part_bytes = WL.part_bytes_per_item;
  if (p.R > 32) {
    set_error("hybrid_decode_fwd: n_q_per_seq * (n_q_heads / n_kv_heads) = %d rows per KV head; at most 32 supported",
              p.R);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  const int nmax = mi > 0x7fffffff ? 0x7fffffff : (int)mi;
  const size_t msm = decode_merge_smem_bytes(p.n_seqs, p.n_qt, p.Hq, p.Hkv, p.window, p.max_ctx_len);
  const int sms = pool->sms;
  // FP8 pools with head_dim 128 may run the tcgen05 kernel of decode_tc.cuh instead of the mma.sync
  // one: environment variable HSWA_DECODE_TC = 1 (full layers) or 2 (every layer), read once per
  // process; unset or 0 keeps decode_kernel, the faster of the two as measured.
  static const int tc_mode = [] {
    const char* e = getenv("HSWA_DECODE_TC");
    return e ? atoi(e) : 0;
  }();
  if (pool->fp8 && Lc.d == 128 && (tc_mode >= 2 || (tc_mode == 1 && p.window <= 0)))
    return launch_tc(p, nmax, sms, msm, stream);
#define HSWA_DEC(DD, MM, F8) launch_t<DD, MM, F8>(p, nmax, sms, msm, stream)
  if (pool->fp8) {
    if (Lc.d == 128) return p.R <= 16 ? HSWA_DEC(128, 1, true) : HSWA_DEC(128, 2, true);
    return p.R <= 16 ? HSWA_DEC(64, 1, true) : HSWA_DEC(64, 2, true);
  }
  if (Lc.d == 128) return p.R <= 16 ? HSWA_DEC(128, 1, false) : HSWA_DEC(128, 2, false);
  return p.R <= 16 ? HSWA_DEC(64, 1, false) : HSWA_DEC(64, 2, false);
#undef HSWA_DEC
}

}  // namespace hswa

// ---------------------------------------------------------------- decode without a workspace

// The scratch of hybrid_decode_fwd_noalloc: one fixed array in device memory, reserved on
// every GPU that loads this library and held until the process exits. Host code cannot use
// this name as a device address; the address is looked up once per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[HSWA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
int noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    hswa::set_error("hybrid_decode_fwd_noalloc: no usable current device (%s)",
                    e == cudaSuccess ? "device index out of range" : cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) {
      hswa::set_error("hybrid_decode_fwd_noalloc: looking up the scratch array failed: %s",
                      cudaGetErrorString(e));
      return HSWA_ERR_CUDA;
    }
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return HSWA_OK;
}
}  // namespace

extern "C" int hybrid_decode_fwd_noalloc(hswa_pool* pool, int layer, const hswa_bf16* q, const hswa_bf16* k_new,
                                         const hswa_bf16* v_new, hswa_bf16* o, int n_seqs, int n_q_per_seq,
                                         const int64_t* ctx_len, int64_t max_ctx_len, const int32_t* seq_ids,
                                         const int32_t* page_table, int pt_stride, int n_q_heads, void* stream) {
  hswa::DecodeLaunch L;
  size_t need = 0;
  // the same argument checks as hybrid_decode_fwd (including that the pool's device is current)
  int rc = hswa::prepare_decode(pool, "hybrid_decode_fwd_noalloc", layer, q, k_new, v_new, o, n_seqs, n_q_per_seq,
                                ctx_len, max_ctx_len, seq_ids, page_table, pt_stride, n_q_heads, &L, &need);
  if (rc || L.n_seqs == 0) return rc;
  if (need > (size_t)HSWA_NOALLOC_SCRATCH_BYTES) {
    hswa::set_error("hybrid_decode_fwd_noalloc: this call needs %zu bytes of scratch but the built-in array holds "
                    "%zu; use hybrid_decode_fwd with a caller-provided workspace",
                    need, (size_t)HSWA_NOALLOC_SCRATCH_BYTES);
    return HSWA_ERR_OUT_OF_MEMORY;
  }
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  L.workspace = scratch;
  L.ws_bytes = (size_t)HSWA_NOALLOC_SCRATCH_BYTES;
  return hswa::launch_decode(L, static_cast<cudaStream_t>(stream));
}

// decode_tc.cuh -- decode over FP8 (E4M3) KV blocks on the 5th-generation tensor cores (tcgen05).
// Included by decode.cu inside its anonymous namespace: the work items, their order (plan_kernel),
// the (m, l, O) partials and merge_kernel are the same as decode_kernel's.
//
// Per block of 128 cached keys of one work item (sequence, split, KV head) and its R <= 32 query
// rows (n_qt tokens x G heads):
//   S^T = K Q^T      M = 128 keys, N = 32 rows, K = 128 dims      (f16 in, f32 accumulate in TMEM)
//   P^T              one thread per key (TMEM lane) holds the key's 32 row scores
//   O^T += V^T P^T   M = 128 dims, N = 32 rows, K = 128 keys      (O^T stays in TMEM for the item)
// Transposing puts the 128 keys of a block (not the 32 rows) on the MMA's M side, so no tile is
// padded. The online softmax keeps one offset per row, identical in every thread; a block's row
// maxima are reduced over its keys only when some score passes its row's offset by more than 2^8
// (the lazy rule of the other kernels), which after the first block of an item is rare.
// The FP8 codes arrive by bulk copies (one KV head's 64 rows of a page are 8 KB of contiguous
// bytes, a ring run is contiguous up to its wrap); four converter warps expand them to f16
// (exact for every E4M3 value) in the 128-byte-swizzled K-major layout the MMAs read. The K scale
// of the KV head folds into the softmax scale and the V scale into O, so nothing else touches the
// tiles. The new tokens' K/V are quantized as the cache will hold them.
// Selected at run time (environment variable HSWA_DECODE_TC = 1: full layers, 2: every layer of an
// FP8 pool with head_dim 128); off by default. Measured on the 256-sequence batch's full layer it takes 12-13 ms against 6.9 ms for
// decode_kernel: per 128-key block the four converter warps need ~1700 clk for K and as much for V
// (eight E4M3 -> f16 conversions per lane per 16 rows), while decode_kernel spreads the same
// conversions over all of its warps. Correct (the FP8 decode tests pass through it) and kept as the
// starting point of a decode whose MMAs read the FP8 codes directly.
// Warps (320 threads): 0-3 softmax and epilogue (thread = TMEM lane: key of a block, then dim of
// O), 4-7 converters and Q staging, 8 producer (work items and their page ids, bulk copies, L2
// prefetch), 9 MMA issuer. Only the producer reads the work list and the page table; the others
// take an item's geometry and page ids from its slot in shared memory.

constexpr int TC_KB = 128;       // keys per block
constexpr int TC_NR = 3;         // stages of raw FP8 codes
constexpr int TC_PREFETCH = 4;   // blocks ahead whose codes the producer pulls into L2
constexpr int TC_THREADS = 320;
constexpr int TC_PRODUCER_WARP = 8;
constexpr int TC_MMA_WARP = 9;
static_assert(SPLIT % TC_KB == 0, "splits of whole 128-key blocks");

struct TcLayout {
  static constexpr int RAW_OFF = 0;               // [TC_NR][K 128 x 128 B | V 128 x 128 B], natural rows
  static constexpr int RAW_STAGE = 2 * TC_KB * 128;
  static constexpr int HALF = TC_KB * 128;        // 128 rows x 64 f16 (one swizzle atom column)
  static constexpr int KC_OFF = RAW_OFF + TC_NR * RAW_STAGE;  // [2 halves][128 keys][128 B] f16 (one buffer:
                                                              // S is done before the next K is converted)
  static constexpr int VC_OFF = KC_OFF + 2 * HALF;            // [2][2 halves][128 keys][128 B] f16
  static constexpr int QHALF = 32 * 128;          // 32 rows x 64 f16
  static constexpr int Q_OFF = VC_OFF + 2 * 2 * HALF;          // [2 halves][32 rows][128 B] f16
  static constexpr int P_OFF = Q_OFF + 2 * QHALF;              // [2][2 halves][32 rows][128 B] f16
  static constexpr int MISC_OFF = P_OFF + 2 * 2 * QHALF;
  static constexpr int BYTES = MISC_OFF + 4096;
  static_assert(BYTES + 1024 <= 227 * 1024, "shared memory per CTA");
};

// A work item's geometry (computed by the producer warp, read by the other roles from its slot).
struct TcItem {
  int item;  // -1: no work left
  int s, g, L, nsp, a, b, n_cached, n_blk;
  int last;
  int ring_ok;  // sliding-window layers: the sequence's ring row id is in range
};

struct TcBars {
  uint64_t item_full[2], item_empty[2];
  uint64_t raw_full[TC_NR], raw_empty[TC_NR];
  uint64_t kc_full, kc_empty, vc_full[2], vc_empty[2];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_free[2], p_full[2], p_free[2];
  uint64_t o_full, o_free;
  uint64_t grp;  // the four softmax warps meet here (a bounded wait, unlike a named barrier)
  uint32_t tmem_base;
  TcItem slot[2];                // the items in flight, published by the producer warp
  int pages[2][SPLIT / 64];      // their page ids (-1: out of range), full layers
  int flags[2][4];
  alignas(16) float red[4][32];  // per-warp row partials (maxima or sums)
  alignas(16) float mo[32];      // row offsets of the item (log2 domain), read as float4
  alignas(16) float al[32];      // factors of the latest offset move, read as float4
  alignas(16) float lt[32];      // row sums of the item
};
static_assert(sizeof(TcBars) <= 4096, "misc region");
static_assert(offsetof(TcBars, mo) % 16 == 0 && offsetof(TcBars, al) % 16 == 0, "float4 reads of the row arrays");
static_assert(TcLayout::MISC_OFF % 1024 == 0, "misc region alignment");


__device__ __forceinline__ void tc_item(const DecParams& p, const WsHeader* hdr, const PlanView& pv, int item,
                                        TcItem& I) {
  I.g = item % p.Hkv;
  const int sc = item / p.Hkv;
  int s, c;
  if (sc < hdr->body_total) {
    int lo = 0, hi = p.n_seqs;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pv.prefix[mid] <= sc) lo = mid; else hi = mid;
    }
    s = pv.order[lo];
    c = sc - pv.prefix[lo];
  } else {
    s = pv.tail[sc - hdr->body_total];
    c = -1;
  }
  I.s = s;
  I.L = (int)safe_len(p, s);
  I.nsp = n_splits(p, I.L);
  if (c < 0) c = I.nsp - 1;
  I.last = c == I.nsp - 1;
  I.a = (int)dec_klo(p, I.L) + c * SPLIT;
  I.b = I.a + SPLIT < I.L ? I.a + SPLIT : I.L;
  I.n_cached = (I.b - I.a + TC_KB - 1) / TC_KB;
  I.n_blk = I.n_cached + (I.last ? 1 : 0);
  I.item = item;
  I.ring_ok = 1;
  if (p.window > 0) {
    const int seq = p.seq_ids[s];
    I.ring_ok = seq >= 0 && seq < p.max_seqs;
  }
}

// Instruction descriptor, kind::f16 with f16 A and B, f32 D (bit layout as idesc_bf16_f32).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Spin until the phase with this parity completes or the time runs out, whatever the error word
// holds (used to let the copies a CTA issued land before it exits).
__device__ __forceinline__ void mbar_wait_quiet(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > limit_ns) return;
}

// One arrival per warp: every lane's prior writes (and fences) are ordered before lane 0's
// release-arrive by the warp barrier. Barriers that a role's four warps signal count 4.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// mbar_wait with one outcome for the whole warp (the softmax warps run warp-wide shuffles and
// votes, so no lane may leave while the others go on).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* err) {
  const bool ok = mbar_wait(bar, parity, err);
  return __all_sync(0xffffffffu, ok);
}

// Four E4M3 codes (bytes of w, lowest first) -> two f16x2 words (exact: every E4M3 value is an
// f16 value).
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
  uint16_t h;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(x));
  return h;
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void sts16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// 32 values per lane, one per row -> the warp's reduction (max or sum over its 32 lanes) of row
// `lane`, by halving exchanges: at each step a lane keeps the half of the rows whose index bit
// matches its own lane bit and receives its partner's values of those rows.
template <bool MAX>
__device__ __forceinline__ float warp_rows_reduce(const float (&x)[32], int lane) {
  float a[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) a[i] = x[i];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float mine = up ? a[i + o] : a[i];
      const float other = up ? a[i] : a[i + o];
      const float recv = __shfl_xor_sync(0xffffffffu, other, o);
      a[i] = MAX ? fmaxf(mine, recv) : mine + recv;
    }
  }
  return a[0];
}

// ---------------------------------------------------------------- roles

// Warp 8: takes work items from the plan's counter and publishes each one (its geometry and, for
// a full layer, its page ids, loaded by the 32 lanes at once) to the other roles; lane 0 then
// copies each cached block's K and V codes into a raw stage and pulls later blocks into L2.
__device__ void tc_producer(const DecParams& p, uint8_t* smem, TcBars* bars) {
  using TL = TcLayout;
  const int lane = threadIdx.x & 31;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  const PlanView pv(p.ws, p.n_seqs);
  const uint32_t raw_base = smem_u32(smem + TL::RAW_OFF);
  uint32_t rawc = 0;
  bool ok = true;
  for (uint32_t it = 0; ok; ++it) {
    const int slot = it & 1;
    if (!warp_wait(&bars->item_empty[slot], ((it >> 1) & 1) ^ 1, p.err)) break;
    int item = 0;
    if (lane == 0) item = atomicAdd(&hdr->counter, 1);
    item = __shfl_sync(0xffffffffu, item, 0);
    const bool done = item >= hdr->total_items;
    TcItem I;
    I.item = -1;
    if (!done) tc_item(p, hdr, pv, item, I);
    int* pages = bars->pages[slot];
    if (!done && p.window <= 0) {
      const int32_t* pt_row = p.page_table ? p.page_table + (int64_t)I.s * p.pt_stride : nullptr;
      const int n_pg = (I.b - I.a + 63) / 64;  // pages of the cached keys (a is a page boundary)
      for (int i = lane; i < n_pg; i += 32) {
        const int lp = I.a / 64 + i;
        const int32_t page = (pt_row && lp < p.pt_stride) ? pt_row[lp] : -1;
        const bool good = page >= 0 && page < p.pages;
        if (!good) record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
        pages[i] = good ? page : -1;
      }
    }
    if (lane == 0) bars->slot[slot] = I;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->item_full[slot]);
    if (done) break;
    if (lane == 0) {
      const uint8_t* kb = p.src_k8;
      const uint8_t* vb = p.src_v8;
      if (p.window > 0) {
        const int64_t row0 = I.ring_ok ? (((int64_t)p.seq_ids[I.s] * p.n_swa + p.ring_layer) * p.Hkv + I.g) * p.window
                                       : 0;
        kb += row0 * 128;
        vb += row0 * 128;
      }
      // the rows of cached block j in up to two contiguous runs: (source byte offset, first
      // destination row, rows); a ring run past the ring's end continues at slot 0
      auto block_runs = [&](int j, int64_t (&src_off)[2], int (&dst_row)[2], int (&nrow)[2]) {
        src_off[0] = src_off[1] = 0;
        dst_row[0] = dst_row[1] = nrow[0] = nrow[1] = 0;
        const int pos0 = I.a + TC_KB * j;
        const int nvalid = I.b - pos0 < TC_KB ? I.b - pos0 : TC_KB;
        if (p.window > 0) {
          if (!I.ring_ok) return;
          const int slot0 = pos0 % p.window;
          const int n1 = nvalid < p.window - slot0 ? nvalid : p.window - slot0;
          src_off[0] = (int64_t)slot0 * 128;
          nrow[0] = n1;
          dst_row[1] = n1;
          nrow[1] = nvalid - n1;
          return;
        }
        for (int h = 0; h < 2; ++h) {
          const int rows = nvalid - 64 * h < 64 ? nvalid - 64 * h : 64;
          if (rows <= 0) break;
          const int page = pages[2 * j + h];
          if (page < 0) continue;
          src_off[h] = ((((int64_t)p.full_layer * p.pages + page) * p.Hkv + I.g) * 64) * 128;
          dst_row[h] = 64 * h;
          nrow[h] = rows;
        }
      };
      // pull block j's codes toward L2 ahead of its copy (the copy then waits on L2, not HBM)
      auto prefetch = [&](int j) {
        int64_t src_off[2];
        int dst_row[2], nrow[2];
        block_runs(j, src_off, dst_row, nrow);
        for (int h = 0; h < 2; ++h) {
          if (nrow[h] <= 0) continue;
          bulk_prefetch_l2(kb + src_off[h], nrow[h] * 128);
          bulk_prefetch_l2(vb + src_off[h], nrow[h] * 128);
        }
      };
      for (int j = 0; j < TC_PREFETCH && j < I.n_cached; ++j) prefetch(j);
      for (int j = 0; j < I.n_cached; ++j, ++rawc) {
        const int st = rawc % TC_NR;
        if (!mbar_wait(&bars->raw_empty[st], ((rawc / TC_NR) & 1) ^ 1, p.err)) {
          ok = false;
          break;
        }
        int64_t src_off[2];
        int dst_row[2], nrow[2];
        block_runs(j, src_off, dst_row, nrow);
        const uint32_t bytes = (uint32_t)(2 * (nrow[0] + nrow[1]) * 128);
        mbar_arrive_expect_tx(&bars->raw_full[st], bytes);
        const uint32_t kdst = raw_base + st * TL::RAW_STAGE;
        for (int h = 0; h < 2; ++h) {
          if (nrow[h] <= 0) continue;
          bulk_g2s(kdst + dst_row[h] * 128, kb + src_off[h], nrow[h] * 128, &bars->raw_full[st]);
          bulk_g2s(kdst + TL::HALF + dst_row[h] * 128, vb + src_off[h], nrow[h] * 128, &bars->raw_full[st]);
        }
        if (j + TC_PREFETCH < I.n_cached) prefetch(j + TC_PREFETCH);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  }
  // let the copies issued last land before this CTA can exit (they have, unless a role timed out)
  if (lane == 0)
    for (uint32_t k = rawc > TC_NR ? rawc - TC_NR : 0; k < rawc; ++k)
      mbar_wait_quiet(&bars->raw_full[k % TC_NR], (k / TC_NR) & 1, 100000000ull);
}

// Warps 4-7: stage each item's Q (f16, swizzled), then expand every block's K and V codes to f16
// tiles (rows past the valid keys, or of a bad page or ring, become zeros).
__device__ void tc_converter(const DecParams& p, uint8_t* smem, TcBars* bars) {
  using TL = TcLayout;
  const int ct = threadIdx.x - 4 * 32;  // 0 .. 127
  const int cw = ct >> 5, lane = ct & 31;
  uint32_t rawc = 0, kvc = 0, qi = 0;
  for (uint32_t it = 0;; ++it) {
    const int slot = it & 1;
    if (!warp_wait(&bars->item_full[slot], (it >> 1) & 1, p.err)) return;
    const TcItem I = bars->slot[slot];
    if (I.item < 0) {
      warp_arrive(&bars->item_empty[slot]);
      return;
    }
    const int* pages = bars->pages[slot];  // held until the item's last block is converted

    // Q rows (row = t * G + hh) as f16, rows >= R zero; the previous item's S MMAs must be done
    if (!warp_wait(&bars->q_empty, (qi & 1) ^ 1, p.err)) return;
    for (int u = ct; u < 32 * 16; u += 128) {
      const int r = u >> 4, ch = u & 15;  // 16-byte f16 chunk ch = dims 8 ch .. 8 ch + 7
      uint4 val = make_uint4(0, 0, 0, 0);
      if (r < p.R) {
        const int t = r / p.G, hh = r - (r / p.G) * p.G;
        const uint4 x = *reinterpret_cast<const uint4*>(
            p.q + (((int64_t)I.s * p.n_qt + t) * p.Hq + I.g * p.G + hh) * 128 + ch * 8);
        val.x = pack_f16x2_sat(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xFFFF0000u));
        val.y = pack_f16x2_sat(__uint_as_float(x.y << 16), __uint_as_float(x.y & 0xFFFF0000u));
        val.z = pack_f16x2_sat(__uint_as_float(x.z << 16), __uint_as_float(x.z & 0xFFFF0000u));
        val.w = pack_f16x2_sat(__uint_as_float(x.w << 16), __uint_as_float(x.w & 0xFFFF0000u));
      }
      *reinterpret_cast<uint4*>(smem + TL::Q_OFF + (ch >> 3) * TL::QHALF + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) =
          val;
    }
    fence_proxy_async_smem();
    warp_arrive(&bars->q_full);
    ++qi;

    const bool ring_ok = I.ring_ok != 0;
    for (int j = 0; j < I.n_blk; ++j, ++kvc) {
      const bool is_new = j >= I.n_cached;
      const int pos0 = is_new ? I.L : I.a + TC_KB * j;
      const int nvalid = is_new ? p.n_qt : (I.b - pos0 < TC_KB ? I.b - pos0 : TC_KB);
      // which rows of the block exist: every page of the item has an entry (-1 when out of range)
      const bool page0_ok = is_new || p.window > 0 || pages[2 * j] >= 0;
      const bool page1_ok = is_new || p.window > 0 || nvalid <= 64 || pages[2 * j + 1] >= 0;
      const uint8_t* raw = smem + TL::RAW_OFF + (rawc % TC_NR) * TL::RAW_STAGE;
      if (!is_new && !warp_wait(&bars->raw_full[rawc % TC_NR], (rawc / TC_NR) & 1, p.err)) return;
      const int b2 = kvc & 1;
      for (int kv = 0; kv < 2; ++kv) {
        // K: one buffer, free once the previous block's S is done; V: two, free once P V is done
        const bool free_ok = kv ? warp_wait(&bars->vc_empty[b2], ((kvc >> 1) & 1) ^ 1, p.err)
                                : warp_wait(&bars->kc_empty, (kvc & 1) ^ 1, p.err);
        if (!free_ok) return;
        uint8_t* dst = smem + (kv ? TL::VC_OFF + b2 * 2 * TL::HALF : TL::KC_OFF);
        // lane (chunk c, row rb + 16 step): each 8-lane phase of a 16-byte access covers chunks 0-3
        // of one row and 4-7 of the next, i.e. eight distinct chunks for the loads and eight
        // distinct swizzled bank groups for the stores
        const int c = lane & 7;  // codes of dims 16 c .. 16 c + 15
        const int rb = cw * 4 + (((lane >> 3) + (c >> 2)) & 3);
        uint4 cd[TC_KB / 16];
        if (!is_new) {
          // all eight loads first (the stage is in bounds whatever rows are valid)
#pragma unroll
          for (int step = 0; step < TC_KB / 16; ++step)
            cd[step] = *reinterpret_cast<const uint4*>(raw + kv * TL::HALF + (step * 16 + rb) * 128 + c * 16);
        } else {
          // the new tokens' rows, quantized with the layer's reciprocal scale as the cache holds them
          const float inv = kv ? p.inv_v[I.g] : p.inv_k[I.g];
          const uint16_t* src_new = kv ? p.v_new : p.k_new;
#pragma unroll
          for (int step = 0; step < TC_KB / 16; ++step) {
            const int r = step * 16 + rb;
            cd[step] = make_uint4(0, 0, 0, 0);
            if (r < nvalid) {
              const uint4* src = reinterpret_cast<const uint4*>(
                  src_new + (((int64_t)I.s * p.n_qt + r) * p.Hkv + I.g) * 128 + c * 16);
              const uint4 x0 = src[0], x1 = src[1];
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
              cd[step] = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
        const int cc = 2 * (c & 3);
#pragma unroll
        for (int step = 0; step < TC_KB / 16; ++step) {
          const int r = step * 16 + rb;
          const bool valid = r < nvalid && (is_new || (p.window > 0 ? ring_ok : (r < 64 ? page0_ok : page1_ok)));
          const uint4 codes = valid ? cd[step] : make_uint4(0, 0, 0, 0);
          uint4 f0, f1;
          e4m3x4_to_f16(codes.x, f0.x, f0.y);
          e4m3x4_to_f16(codes.y, f0.z, f0.w);
          e4m3x4_to_f16(codes.z, f1.x, f1.y);
          e4m3x4_to_f16(codes.w, f1.z, f1.w);
          uint8_t* row = dst + (c >> 2) * TL::HALF + r * 128;
          *reinterpret_cast<uint4*>(row + ((cc ^ (r & 7)) << 4)) = f0;
          *reinterpret_cast<uint4*>(row + (((cc + 1) ^ (r & 7)) << 4)) = f1;
        }
        fence_proxy_async_smem();
        warp_arrive(kv ? &bars->vc_full[b2] : &bars->kc_full);
      }
      if (!is_new) {
        warp_arrive(&bars->raw_empty[rawc % TC_NR]);
        ++rawc;
      }
    }
    warp_arrive(&bars->item_empty[slot]);
  }
}

// Warp 9, lane 0: S^T of each block as soon as its K tile is ready, then O^T += V^T P^T of the
// block before it once its P is written, so a block's softmax overlaps the previous P V.
__device__ void tc_mma(const DecParams& p, uint8_t* smem, TcBars* bars, uint32_t tbase) {
  using TL = TcLayout;
  constexpr uint32_t IDESC_S = idesc_f16_f32(128, 32, false, false);
  constexpr uint32_t IDESC_PV = idesc_f16_f32(128, 32, true, false);
  const uint32_t kc_base = smem_u32(smem + TL::KC_OFF);
  const uint32_t vc_base = smem_u32(smem + TL::VC_OFF);
  const uint32_t q_base = smem_u32(smem + TL::Q_OFF);
  const uint32_t p_base = smem_u32(smem + TL::P_OFF);
  const uint32_t o_tmem = tbase + 64;
  uint32_t kvc = 0, sc = 0, pc = 0, qi = 0, oi = 0;

  auto issue_pv = [&](uint32_t kvj, bool first) -> bool {
    const uint32_t pb = pc & 1;
    if (!mbar_wait(&bars->p_full[pb], (pc >> 1) & 1, p.err)) return false;
    if (!mbar_wait(&bars->vc_full[kvj & 1], (kvj >> 1) & 1, p.err)) return false;
    if (first && !mbar_wait(&bars->o_free, (oi & 1) ^ 1, p.err)) return false;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < TC_KB / 16; ++kk) {
      // A = V^T (dims x keys, MN-major: each key row holds 64 dims per half), B = P (rows x keys)
      const uint64_t adesc = smem_desc_sw128(vc_base + (kvj & 1) * 2 * TL::HALF + kk * 16 * 128, TL::HALF, 1024);
      const uint64_t bdesc = smem_desc_sw128(p_base + pb * 2 * TL::QHALF + (kk >> 2) * TL::QHALF + (kk & 3) * 32, 16,
                                             1024);
      umma_ss(o_tmem, adesc, bdesc, IDESC_PV, (!first || kk > 0) ? 1u : 0u);
    }
    umma_commit(&bars->p_free[pb]);
    umma_commit(&bars->vc_empty[kvj & 1]);
    ++pc;
    return true;
  };

  for (uint32_t it = 0;; ++it) {
    const int slot = it & 1;
    if (!mbar_wait(&bars->item_full[slot], (it >> 1) & 1, p.err)) return;
    const TcItem I = bars->slot[slot];
    mbar_arrive(&bars->item_empty[slot]);
    if (I.item < 0) return;
    if (!mbar_wait(&bars->q_full, qi & 1, p.err)) return;
    const uint32_t kv0 = kvc;
    for (int j = 0; j < I.n_blk; ++j, ++kvc) {
      if (!mbar_wait(&bars->kc_full, kvc & 1, p.err)) return;
      const uint32_t sb = sc & 1;
      if (!mbar_wait(&bars->s_free[sb], ((sc >> 1) & 1) ^ 1, p.err)) return;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 128 / 16; ++kk) {
        const uint32_t off = (kk >> 2) * TL::HALF + (kk & 3) * 32;
        const uint64_t adesc = smem_desc_sw128(kc_base + off, 16, 1024);
        const uint64_t bdesc = smem_desc_sw128(q_base + (kk >> 2) * TL::QHALF + (kk & 3) * 32, 16, 1024);
        umma_ss(tbase + sb * 32, adesc, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
      }
      umma_commit(&bars->s_full[sb]);
      umma_commit(&bars->kc_empty);
      ++sc;
      if (j == I.n_blk - 1) {
        umma_commit(&bars->q_empty);  // every S of the item is issued: Q may be restaged once they finish
        ++qi;
      }
      if (j > 0 && !issue_pv(kv0 + j - 1, j == 1)) return;
    }
    if (!issue_pv(kv0 + I.n_blk - 1, I.n_blk == 1)) return;
    umma_commit(&bars->o_full);
    ++oi;
  }
}

// Warps 0-3: softmax of every block (thread = key), then the item's epilogue (thread = dim). The
// row offsets live in shared memory (the same for every thread): lane r of warp 0 moves row r's.
__device__ void tc_softmax(const DecParams& p, uint8_t* smem, TcBars* bars, uint32_t tbase) {
  using TL = TcLayout;
  const int t = threadIdx.x;  // 0 .. 127
  const int w = t >> 5, lane = t & 31;
  const uint32_t trow = tbase + ((uint32_t)(w * 32) << 16);
  const uint32_t p_base = smem_u32(smem + TL::P_OFF);
  uint32_t sc = 0, pc = 0, oi = 0, gs = 0;
  // all four warps arrive; false when the wait ran out (every warp then leaves)
  auto group_sync = [&]() -> bool {
    warp_arrive(&bars->grp);
    return warp_wait(&bars->grp, (gs++) & 1, p.err);
  };
  for (uint32_t it = 0;; ++it) {
    const int slot = it & 1;
    if (!warp_wait(&bars->item_full[slot], (it >> 1) & 1, p.err)) return;
    const TcItem I = bars->slot[slot];
    warp_arrive(&bars->item_empty[slot]);
    if (I.item < 0) return;
    const int item = I.item;
    const float sl2 = p.scale_log2 * p.k_scale[I.g];  // the K scale of an FP8 pool folds in here
    float l_part[32];
#pragma unroll
    for (int r = 0; r < 32; ++r) l_part[r] = 0.f;
    for (int j = 0; j < I.n_blk; ++j) {
      const bool is_new = j >= I.n_cached;
      const int pos0 = is_new ? I.L : I.a + TC_KB * j;
      const int nvalid = is_new ? p.n_qt : (I.b - pos0 < TC_KB ? I.b - pos0 : TC_KB);
      const uint32_t sb = sc & 1;
      if (!warp_wait(&bars->s_full[sb], (sc >> 1) & 1, p.err)) return;
      tc_fence_after();
      float x[32];
      tmem_ld32(trow + sb * 32, reinterpret_cast<uint32_t(&)[32]>(x));
      tmem_wait_ld();
      tc_fence_before();
      warp_arrive(&bars->s_free[sb]);
      ++sc;
      const bool need_mask = is_new || nvalid < TC_KB || (p.window > 0 && pos0 < I.L + p.n_qt - p.window);
      if (need_mask) {
        // rows of this key: token t sees cached key kp when kp >= L + t - W + 1 (sliding window),
        // new key L + k when k <= t; rows r = t G + hh
        int r_lo = 32, r_hi = -1;
        if (t < nvalid) {
          const int dk = pos0 + t - I.L;  // < 0 for cached keys
          const int t_lo = dk > 0 ? dk : 0;
          int t_hi = 32;
          if (p.window > 0) t_hi = dk + p.window - 1 < 32 ? dk + p.window - 1 : 32;
          r_lo = t_lo * p.G;
          r_hi = t_hi < 0 ? -1 : (t_hi + 1) * p.G - 1;
        }
#pragma unroll
        for (int r = 0; r < 32; ++r) x[r] = (r >= r_lo && r <= r_hi) ? x[r] * sl2 : -INFINITY;
      } else {
#pragma unroll
        for (int r = 0; r < 32; ++r) x[r] *= sl2;
      }
      // does any score pass its row's offset by more than 2^8? (always at an item's first block)
      bool up = j == 0;
      if (!up) {
#pragma unroll
        for (int r4 = 0; r4 < 32; r4 += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(&bars->mo[r4]);
          up |= x[r4] > m4.x + 8.f;
          up |= x[r4 + 1] > m4.y + 8.f;
          up |= x[r4 + 2] > m4.z + 8.f;
          up |= x[r4 + 3] > m4.w + 8.f;
        }
      }
      up = __any_sync(0xffffffffu, up);
      if (lane == 0) bars->flags[j & 1][w] = up ? 1 : 0;
      if (!group_sync()) return;
      const bool any = (bars->flags[j & 1][0] | bars->flags[j & 1][1] | bars->flags[j & 1][2] |
                        bars->flags[j & 1][3]) != 0;
      if (any) {
        // the block's row maxima; a row whose maximum passed its offset moves the offset there
        bars->red[w][lane] = warp_rows_reduce<true>(x, lane);
        if (!group_sync()) return;
        if (w == 0) {
          const float mb = fmaxf(fmaxf(bars->red[0][lane], bars->red[1][lane]),
                                 fmaxf(bars->red[2][lane], bars->red[3][lane]));
          const float old = j == 0 ? -INFINITY : bars->mo[lane];
          float al = 1.f;
          if (mb > old + 8.f) {
            al = ex2_approx(old - mb);  // 0 when the old offset is -inf
            bars->mo[lane] = mb;
          } else if (j == 0) {
            bars->mo[lane] = old;  // -inf: no key of this row yet
          }
          bars->al[lane] = al;
          const bool moved = __any_sync(0xffffffffu, al != 1.f);
          if (lane == 0) bars->flags[j & 1][0] = moved ? 2 : 0;
        }
        if (!group_sync()) return;
        if (bars->flags[j & 1][0] == 2 && j > 0) {
#pragma unroll
          for (int r4 = 0; r4 < 32; r4 += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(&bars->al[r4]);
            l_part[r4] *= a4.x;
            l_part[r4 + 1] *= a4.y;
            l_part[r4 + 2] *= a4.z;
            l_part[r4 + 3] *= a4.w;
          }
          // O^T holds the item's earlier blocks: rescale its columns once the last P V is done
          const uint32_t pp = pc - 1;
          if (!warp_wait(&bars->p_free[pp & 1], (pp >> 1) & 1, p.err)) return;
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {  // 16 columns at a time (register pressure)
            uint32_t o[16];
            tmem_ld16(trow + 64 + 16 * h, o);
            tmem_wait_ld();
#pragma unroll
            for (int r = 0; r < 16; ++r) o[r] = __float_as_uint(__uint_as_float(o[r]) * bars->al[16 * h + r]);
            tmem_st16(trow + 64 + 16 * h, o);
          }
          tmem_wait_st();
        }
      }
      // P^T of this key: 2^(x - offset), f16, into row r of the P tile (keys along the row)
      const uint32_t pb = pc & 1;
      if (!warp_wait(&bars->p_free[pb], ((pc >> 1) & 1) ^ 1, p.err)) return;
      const uint32_t pcol = p_base + pb * 2 * TL::QHALF + (t >> 6) * TL::QHALF + (t & 7) * 2;
      const int chunk = (t & 63) >> 3;
#pragma unroll
      for (int r4 = 0; r4 < 32; r4 += 4) {
        const float4 m4 = *reinterpret_cast<const float4*>(&bars->mo[r4]);
        const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
        float pr[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float moff = mv[q] == -INFINITY ? 0.f : mv[q];
          pr[q] = ex2_approx(x[r4 + q] - moff);
          l_part[r4 + q] += pr[q];
        }
#pragma unroll
        for (int q = 0; q < 4; q += 2) {  // rows r, r + 1 of this key: one conversion, two stores
          const uint32_t h2 = pack_f16x2_sat(pr[q], pr[q + 1]);
          const int r = r4 + q;
          sts16(pcol + r * 128 + ((chunk ^ (r & 7)) << 4), (uint16_t)(h2 & 0xFFFFu));
          sts16(pcol + (r + 1) * 128 + ((chunk ^ ((r + 1) & 7)) << 4), (uint16_t)(h2 >> 16));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&bars->p_full[pb]);
      ++pc;
    }

    // ---- epilogue: row sums, then O^T (thread = dim) scaled and written
    bars->red[w][lane] = warp_rows_reduce<false>(l_part, lane);
    if (!group_sync()) return;
    if (w == 0) bars->lt[lane] = (bars->red[0][lane] + bars->red[1][lane]) + (bars->red[2][lane] + bars->red[3][lane]);
    if (!group_sync()) return;
    if (!warp_wait(&bars->o_full, oi & 1, p.err)) return;
    ++oi;
    tc_fence_after();
    uint32_t o[32];
    tmem_ld32(trow + 64, o);
    tmem_wait_ld();
    tc_fence_before();
    warp_arrive(&bars->o_free);
    const float vs = p.v_scale[I.g];  // the V scale of an FP8 pool multiplies O
    const int d = t;
    if (I.nsp == 1) {
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        if (r < p.R) {
          const int tt = r / p.G, hh = r - (r / p.G) * p.G;
          const float val = __uint_as_float(o[r]) * (vs / bars->lt[r]);
          p.o[(((int64_t)I.s * p.n_qt + tt) * p.Hq + I.g * p.G + hh) * 128 + d] = f32_to_bf16(val);
        }
      }
    } else {
      float* part = reinterpret_cast<float*>(p.ws + p.part_off + (size_t)item * p.part_bytes);
#pragma unroll
      for (int r = 0; r < 32; ++r)
        if (r < p.R) part[r * 128 + d] = __uint_as_float(o[r]) * vs;
      if (t < p.R) {
        part[p.R * 128 + t] = bars->mo[t];
        part[p.R * 128 + p.R + t] = bars->lt[t];
      }
    }
  }
}

__global__ void __launch_bounds__(TC_THREADS, 1) decode_tc_kernel(const __grid_constant__ DecParams p) {
  using TL = TcLayout;
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  TcBars* bars = reinterpret_cast<TcBars*>(smem + TL::MISC_OFF);
  const int warp = threadIdx.x >> 5;
  if (read_error(p.err) != 0) return;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->item_full[i], 1);
      mbar_init(&bars->item_empty[i], 1 + 4 + 4);  // the MMA thread, the softmax and converter warps
      mbar_init(&bars->vc_full[i], 4);
      mbar_init(&bars->vc_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 4);
      mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->p_free[i], 1);
    }
    for (int i = 0; i < TC_NR; ++i) {
      mbar_init(&bars->raw_full[i], 1);
      mbar_init(&bars->raw_empty[i], 4);
    }
    mbar_init(&bars->kc_full, 4);
    mbar_init(&bars->kc_empty, 1);
    mbar_init(&bars->q_full, 4);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_free, 4);
    mbar_init(&bars->grp, 4);
    fence_barrier_init();
  }
  if (warp == TC_MMA_WARP) {
    tmem_alloc(&bars->tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;

  if (warp < 4) {
    tc_softmax(p, smem, bars, tbase);
  } else if (warp < 8) {
    tc_converter(p, smem, bars);
  } else if (warp == TC_PRODUCER_WARP) {
    tc_producer(p, smem, bars);
  } else {
    if ((threadIdx.x & 31) == 0) tc_mma(p, smem, bars, tbase);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == TC_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, 128);
  }
}

// prefill_narrow.cu -- causal sliding-window prefill for narrow windows (W <= 129), where the
// band of every 128-row query tile lies in two 128-key tiles.
//
// Math ("Sliding Window Attention (SWA) no riron to jisso", section "formal definition",
// eqs. (1)-(5)): query i attends keys j in [max(0, i - W + 1), i] with weights
// softmax_j(q_i . k_j / sqrt(d)) on v_j; query head h reads KV head h / G (section
// "Mistral: SWA and GQA"). Tiles outside the band are never loaded (section "sparsity:
// Flash Attention and BlockSparse").
//
// Work unit = (query tile t, batch row b, KV head g). Key tiles t - 1 (the rolling buffer when it
// lies before the chunk, zeros before position 0) and t are loaded once per unit and stay in
// shared memory while the G query heads of KV head g stream through two slots (slot q takes heads
// q, q + 2, ... of the group). One head is one pass over both key tiles:
//   S = Q [K_{t-1}; K_t]^T     one N = 256 MMA chain into the slot's 256 TMEM columns;
//   one softmax over the band  row r of the tile keeps S columns [i - W + 1 - kb0, i - kb0]
//                              (kb0 = position of column 0), which for warp w (rows 32w .. 32w+31)
//                              lie in 32-column chunks w .. w + 4: only those five are read, and
//                              with W = 128 away from the sequence start the band edge is the lane
//                              index in chunks w and w + 4 and the three between are whole;
//   P (bf16) over S's first 128 columns, O += P [V_{t-1}; V_t] into columns 128 .. 128 + D.
// No online rescaling (one softmax step per head) and two hand-offs per head.
//   warps 0-3 / 4-7  softmax + epilogue of slot 0 / slot 1 (one thread per TMEM lane)
//   warp 8           K/V producer: both K tiles, then both V tiles of a unit (TMA; the rolling
//                    buffer by TMA when W = 128 and the chunk starts on a tile boundary, else
//                    cp.async, or a dequantizing loader for FP8 pools)
//   warp 9           MMA issuer for both slots (S of both slots, then P V of both); owns TMEM
//   warp 10          Q producer: a slot's next head loads as soon as its S has read the Q tile
//   warp 11          completes the warpgroup
// TMEM: slot q owns columns [256 q, 256 q + 256).
// Shared memory: Q 2 tiles, K [D / 64 blocks][256 rows][128 B] (tile t - 1 then tile t, so one
// MMA reads 256 keys), V 2 tiles, output staging 32 KB.
#include "common.cuh"
#include "internal.h"
#include "prefill_tile.cuh"

namespace hswa {

namespace {

constexpr int NSLOT = 2;          // query-head slots
constexpr int NWARPS = 12;
constexpr int NTHREADS = NWARPS * 32;
constexpr int KV_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int QP_WARP = 10;

struct NParams {
  int B, n_q, Hq, Hkv, G;
  int window;  // 1 .. BN + 1
  const int64_t* start_pos;
  const int32_t* seq_ids;
  const uint16_t* ring_k;
  const uint16_t* ring_v;
  const uint8_t* ring_k8;  // FP8 pools: the rings as E4M3 codes, and this layer's per-KV-head scales
  const uint8_t* ring_v8;
  const float* k_scale;
  const float* v_scale;
  int fp8;
  int ring_layer, n_swa, max_seqs, ring_tma;
  float scale_log2;
  int n_tiles;  // query tiles per batch row
  int n_units;  // n_tiles * B * Hkv
  int64_t max_start;
  int* err;
};

template <int D>
struct NLayout {
  static constexpr int BLOCK = BM * 128;         // [128 rows][64 elems] swizzled = 16 KB
  static constexpr int TILE = BLOCK * (D / 64);  // one 128 x D tile
  static constexpr int KBLK = 2 * BLOCK;         // one 64-dim block of the 256-key K operand
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NSLOT * TILE;
  static constexpr int V_OFF = K_OFF + 2 * TILE;
  static constexpr int O_OFF = V_OFF + 2 * TILE;  // 4 KB output staging per softmax warp
  static constexpr int BAR_OFF = O_OFF + 2 * BLOCK;
  static constexpr int BYTES = BAR_OFF + 256;
  static_assert(BYTES + 1024 <= 227 * 1024, "shared memory per CTA");
  static constexpr int O_COL = 128;  // O within a slot's TMEM columns
};

struct NBars {
  uint64_t q_full[NSLOT], q_empty[NSLOT];
  uint64_t k_full, k_empty, v_full, v_empty;
  uint64_t s_full[NSLOT], p_full[NSLOT], o_full[NSLOT], o_free[NSLOT];
  uint32_t tmem_base;
};

struct NGeo {
  int t, b, g, P;
  int i0;         // absolute position of the tile's first row
  int nh[NSLOT];  // heads of each slot
};

__device__ __forceinline__ void make_ngeo(const NParams& p, int unit, NGeo& G) {
  const int per_t = p.B * p.Hkv;
  G.t = unit / per_t;
  const int rem = unit - G.t * per_t;
  G.b = rem / p.Hkv;
  G.g = rem - G.b * p.Hkv;
  int64_t P = p.start_pos ? p.start_pos[G.b] : 0;
  if (P < 0 || P > p.max_start) {  // positions must stay below 2^31
    record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
    P = 0;
  }
  G.P = (int)P;
  G.i0 = G.P + G.t * BM;
  G.nh[0] = (p.G + 1) / 2;
  G.nh[1] = p.G / 2;
}

// ---------------------------------------------------------------- one softmax pass per head

// Row r of the tile at position i keeps S columns [c_lo, c_hi] of the 256 (column c = position
// kb0 + c); warp w's rows need chunks w .. w + 4 only. FAST: W = 128 with no window clipped at
// position 0, where c_lo = r + 1 and c_hi = r + 128, so chunk w keeps lanes j > lane, chunk w + 4
// keeps j <= lane and chunks w + 1 .. w + 3 are whole. P = 2^(s * sl2 - m) (bf16) goes to the
// chunk's 16 P columns (zeros for the chunks outside the five); returns the row sum.
template <bool FAST>
__device__ __forceinline__ float softmax_band(uint32_t trow, uint32_t s_col, int w, float sl2, int c_lo, int c_hi) {
  const int lane = threadIdx.x & 31;
  uint32_t v[160];
  tmem_ld32_into<0>(trow + s_col + 32 * (w + 0), v);
  tmem_ld32_into<32>(trow + s_col + 32 * (w + 1), v);
  tmem_ld32_into<64>(trow + s_col + 32 * (w + 2), v);
  tmem_ld32_into<96>(trow + s_col + 32 * (w + 3), v);
  tmem_ld32_into<128>(trow + s_col + 32 * (w + 4), v);
  tmem_wait_ld();
  reg_fence_into<0>(v);
  reg_fence_into<32>(v);
  reg_fence_into<64>(v);
  reg_fence_into<96>(v);
  reg_fence_into<128>(v);
  if (FAST) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j <= lane) v[j] = 0xFF800000u;
      if (j > lane) v[128 + j] = 0xFF800000u;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 5; ++c)
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = 32 * (w + c) + j;
        if (col < c_lo || col > c_hi) v[32 * c + j] = 0xFF800000u;
      }
  }
  float m0 = __uint_as_float(v[0]), m1 = __uint_as_float(v[1]);
#pragma unroll
  for (int k = 2; k < 160; k += 4) {
    m0 = fmax3(m0, __uint_as_float(v[k]), __uint_as_float(v[k + 1]));
    m1 = fmax3(m1, __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
  }
  const float mx = fmaxf(m0, m1);
  const float moff = mx == -INFINITY ? 0.f : mx * sl2;
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t neg2 = f2_pack(-moff, -moff);
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int c = 0; c < 5; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
      const uint64_t x =
          f2_fma(f2_pack(__uint_as_float(v[32 * c + k]), __uint_as_float(v[32 * c + k + 1])), scale2, neg2);
      float x0, x1;
      f2_unpack(x, x0, x1);
      const uint64_t e = f2_pack(ex2_approx(x0), ex2_approx(x1));
      acc[(k >> 1) & 3] = f2_add(acc[(k >> 1) & 3], e);
      float e0, e1;
      f2_unpack(e, e0, e1);
      pk[k >> 1] = pack_bf16x2(e0, e1);
    }
    tmem_st16(trow + s_col + 16 * (w + c), pk);
  }
  uint32_t z[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) z[k] = 0u;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (k < w || k > w + 4) tmem_st16(trow + s_col + 16 * k, z);
  float a0, a1, b0, b1, c0, c1, d0, d1;
  f2_unpack(acc[0], a0, a1);
  f2_unpack(acc[1], b0, b1);
  f2_unpack(acc[2], c0, c1);
  f2_unpack(acc[3], d0, d1);
  return ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
}

// ---------------------------------------------------------------- K/V producer

template <int D>
__device__ void kv_producer(const NParams& p, uint8_t* smem, NBars* bars, const CUtensorMap* tm_k,
                            const CUtensorMap* tm_v, const CUtensorMap* tm_rk, const CUtensorMap* tm_rv) {
  using L = NLayout<D>;
  const int lane = threadIdx.x & 31;
  uint32_t nu = 0;  // units loaded (k_empty / v_empty phase)
  for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x, ++nu) {
    NGeo G;
    make_ngeo(p, unit, G);
    const int seq = p.seq_ids ? p.seq_ids[G.b] : 0;
    const bool seq_ok = seq >= 0 && seq < p.max_seqs;
    const int64_t ring_row = seq_ok ? ((int64_t)seq * p.n_swa + p.ring_layer) * p.Hkv + G.g : 0;
    const bool ring_fast = p.ring_tma && (G.P % BN) == 0;
    const int j0 = G.t - 1;                                  // key tile t - 1 (jj = 0) and t (jj = 1)
    const bool ring_tile = j0 < 0 && p.start_pos != nullptr;  // tile t - 1 lies in the rolling buffer
    for (int kv = 0; kv < 2; ++kv) {
      uint64_t* full = kv ? &bars->v_full : &bars->k_full;
      if (!mbar_wait(kv ? &bars->v_empty : &bars->k_empty, (nu & 1) ^ 1, p.err)) return;
      const CUtensorMap* tm = kv ? tm_v : tm_k;
      // K: the two tiles are rows 0..127 and 128..255 of each 64-dim block; V: two separate tiles
      const int blk_stride = kv ? L::BLOCK : L::KBLK;
      uint8_t* dst0 = smem + (kv ? L::V_OFF : L::K_OFF);
      uint8_t* dst1 = dst0 + (kv ? L::TILE : L::BLOCK);
      if (ring_tile && !ring_fast) {
        // rows of the ring one by one (zeros where the ring holds nothing), before the TMA part
        if (!seq_ok && lane == 0) record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
        const int held_lo = (G.P - p.window > 0) ? G.P - p.window : 0;
        const int64_t base = ring_row * p.window * D;
        if (p.fp8)
          ring_rows_fp8<D>((kv ? p.ring_v8 : p.ring_k8) + base, seq_ok, held_lo, G.P, p.window,
                           kv ? p.v_scale[G.g] : p.k_scale[G.g], dst0, G.P + BN * j0, lane, blk_stride);
        else
          ring_rows_cpasync<D>((kv ? p.ring_v : p.ring_k) + base, seq_ok, held_lo, G.P, p.window, dst0,
                               G.P + BN * j0, lane, blk_stride);
      }
      if (lane == 0) {
        const bool tile0_tma = !(ring_tile && !ring_fast);
        mbar_arrive_expect_tx(full, (tile0_tma ? 2 : 1) * L::TILE);
        if (tile0_tma) {
          if (ring_tile) {
            // W = 128 and the chunk starts on a tile boundary: the tile is one box of the ring
            if (!seq_ok) record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
            // a tile wholly before position 0 (P = 0) is read outside the map: zero fill
            const int slot = (G.P + BN * j0) % p.window;
            const int row = (seq_ok && G.P + BN * j0 >= 0) ? (int)ring_row : -1;
            for (int dh = 0; dh < D / 64; ++dh)
              tma_load_3d(dst0 + dh * blk_stride, kv ? tm_rv : tm_rk, full, dh * 64, slot, row);
          } else {
            // chunk rows (tile -1 of a chunk without a prefix lies before row 0: zero fill)
            for (int dh = 0; dh < D / 64; ++dh)
              tma_load_4d(dst0 + dh * blk_stride, tm, full, dh * 64, G.g, BN * j0, G.b);
          }
        }
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_4d(dst1 + dh * blk_stride, tm, full, dh * 64, G.g, BN * G.t, G.b);
      }
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------- Q producer

template <int D>
__device__ void q_producer(const NParams& p, uint8_t* smem, NBars* bars, const CUtensorMap* tm_q) {
  using L = NLayout<D>;
  uint32_t nq[NSLOT] = {0, 0};
  for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x) {
    NGeo G;
    make_ngeo(p, unit, G);
    const int nk = G.nh[0] > G.nh[1] ? G.nh[0] : G.nh[1];
    for (int k = 0; k < nk; ++k) {
#pragma unroll
      for (int q = 0; q < NSLOT; ++q) {
        if (k >= G.nh[q]) continue;
        // the slot's Q buffer is free once the S of its previous head has completed
        if (!mbar_wait(&bars->q_empty[q], (nq[q] & 1) ^ 1, p.err)) return;
        ++nq[q];
        const int h = G.g * p.G + q + 2 * k;
        mbar_arrive_expect_tx(&bars->q_full[q], L::TILE);
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_4d(smem + L::Q_OFF + q * L::TILE + dh * L::BLOCK, tm_q, &bars->q_full[q], dh * 64, h,
                      G.t * BM, G.b);
      }
    }
  }
}

// ---------------------------------------------------------------- MMA issuer (both slots)

// Per head k: S of both slots (each after its Q landed and its previous O was read out), then
// P V of both (each after its softmax). While one slot's softmax or epilogue runs, the tensor
// core works on the other slot.
template <int D>
__device__ void mma_issuer(const NParams& p, uint8_t* smem, NBars* bars, uint32_t tbase) {
  using L = NLayout<D>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, 2 * BN, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
  const uint32_t q_base = smem_u32(smem + L::Q_OFF);
  const uint32_t k_base = smem_u32(smem + L::K_OFF);
  const uint32_t v_base = smem_u32(smem + L::V_OFF);
  uint32_t nqf = 0;  // bit q: q_full phase of slot q
  uint32_t np = 0;   // bit q: p_full phase
  uint32_t nof = 0;  // bit q: o_free phase (the slot's previous O has been read)
  uint32_t nu = 0;   // units (k_full / v_full phase)

  for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x, ++nu) {
    NGeo G;
    make_ngeo(p, unit, G);
    if (!mbar_wait(&bars->k_full, nu & 1, p.err)) return;
    tc_fence_after();
    const int nk = G.nh[0] > G.nh[1] ? G.nh[0] : G.nh[1];
    for (int k = 0; k < nk; ++k) {
#pragma unroll
      for (int q = 0; q < NSLOT; ++q) {
        if (k >= G.nh[q]) continue;
        if (!mbar_wait(&bars->q_full[q], (nqf >> q) & 1u, p.err)) return;
        nqf ^= 1u << q;
        if (!mbar_wait(&bars->o_free[q], ((nof >> q) & 1u) ^ 1u, p.err)) return;
        nof ^= 1u << q;
        tc_fence_after();
        const uint32_t qb = q_base + q * L::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = (kk >> 2) * L::BLOCK + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * L::KBLK + (kk & 3) * 32;
          umma_ss(tbase + 256 * q, smem_desc_sw128(qb + qoff, 16, 1024), smem_desc_sw128(k_base + koff, 16, 1024),
                  IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[q]);
        umma_commit(&bars->q_empty[q]);  // this head's Q tile is read
      }
      if (k == nk - 1) umma_commit(&bars->k_empty);  // every S of the unit is issued
      if (k == 0) {
        if (!mbar_wait(&bars->v_full, nu & 1, p.err)) return;
        tc_fence_after();
      }
#pragma unroll
      for (int q = 0; q < NSLOT; ++q) {
        if (k >= G.nh[q]) continue;
        if (!mbar_wait(&bars->p_full[q], (np >> q) & 1u, p.err)) return;
        np ^= 1u << q;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 2 * BN / 16; ++kk) {
          const uint64_t bdesc =
              smem_desc_sw128(v_base + (kk >> 3) * L::TILE + (kk & 7) * 16 * 128, L::BLOCK, 1024);
          umma_ts(tbase + 256 * q + L::O_COL, tbase + 256 * q + kk * 8, bdesc, IDESC_PV, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->o_full[q]);
      }
    }
    umma_commit(&bars->v_empty);  // every P V of the unit is issued
  }
}

// ---------------------------------------------------------------- softmax + epilogue (one per slot)

template <int D>
__device__ void softmax_slot(const NParams& p, uint8_t* smem, NBars* bars, uint32_t tbase, const int q,
                             const CUtensorMap* tm_o) {
  using L = NLayout<D>;
  const int wq = (threadIdx.x >> 5) & 3;
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;
  const uint32_t trow = tbase + ((uint32_t)(wq * 32) << 16);
  const uint32_t s_col = 256 * q;
  const float sl2 = p.scale_log2;
  uint8_t* stage = smem + L::O_OFF + q * L::BLOCK + wq * 4096;
  uint32_t ns = 0;  // heads whose S arrived (s_full phase)
  uint32_t no = 0;  // heads whose O arrived (o_full phase)

  for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x) {
    NGeo G;
    make_ngeo(p, unit, G);
    const int kb0 = G.P + BN * (G.t - 1);  // position of S column 0
    const int i = G.i0 + r;
    const int lo_i = (i - p.window + 1 > 0) ? i - p.window + 1 : 0;
    const int c_lo = lo_i - kb0, c_hi = i - kb0;
    const bool fast = p.window == 128 && G.i0 >= 127;
    for (int k = 0; k < G.nh[q]; ++k) {
      if (!mbar_wait(&bars->s_full[q], ns & 1, p.err)) return;
      ++ns;
      tc_fence_after();
      const float l = fast ? softmax_band<true>(trow, s_col, wq, sl2, c_lo, c_hi)
                           : softmax_band<false>(trow, s_col, wq, sl2, c_lo, c_hi);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[q]);
      if (!mbar_wait(&bars->o_full[q], no & 1, p.err)) return;
      ++no;
      tc_fence_after();
      // O leaves TMEM first: the slot's next S may overwrite its columns while it is stored
      store_output_release<D>(trow, s_col + L::O_COL, l, stage, lane, tm_o, G.g * p.G + q + 2 * k,
                              G.t * BM + wq * 32, G.b, p.n_q, &bars->o_free[q]);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_narrow_kernel(const __grid_constant__ NParams p, const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_rk, const __grid_constant__ CUtensorMap tm_rv,
                          const __grid_constant__ CUtensorMap tm_o) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  NBars* bars = reinterpret_cast<NBars*>(smem + NLayout<D>::BAR_OFF);
  const int warp = threadIdx.x >> 5;

  if (read_error(p.err) != 0) return;  // a pending device error: skip the work

  if (threadIdx.x == 0) {
    for (int q = 0; q < NSLOT; ++q) {
      mbar_init(&bars->q_full[q], 1);
      mbar_init(&bars->q_empty[q], 1);
      mbar_init(&bars->s_full[q], 1);
      mbar_init(&bars->p_full[q], 128);
      mbar_init(&bars->o_full[q], 1);
      mbar_init(&bars->o_free[q], 128);
    }
    mbar_init(&bars->k_full, 1);
    mbar_init(&bars->k_empty, 1);
    mbar_init(&bars->v_full, 1);
    mbar_init(&bars->v_empty, 1);
    fence_barrier_init();
  }
  if (warp == KV_WARP && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == MMA_WARP) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 " HSWA_STR(HSWA_SOFTMAX_REGS) ";" ::: "memory");
    softmax_slot<D>(p, smem, bars, tbase, warp >> 2, &tm_o);
    if ((threadIdx.x & 31) == 0) bulk_wait_all();  // output stores complete before the CTA exits
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 " HSWA_STR(HSWA_PRODUCER_REGS) ";" ::: "memory");
    if (warp == KV_WARP) {
      kv_producer<D>(p, smem, bars, &tm_k, &tm_v, &tm_rk, &tm_rv);
    } else if ((threadIdx.x & 31) == 0) {
      if (warp == MMA_WARP) mma_issuer<D>(p, smem, bars, tbase);
      else if (warp == QP_WARP) q_producer<D>(p, smem, bars, &tm_q);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace

int launch_prefill_narrow(const PrefillLaunch& Lc, cudaStream_t stream) {
  const hswa_pool* pool = Lc.pool;
  const hswa_pool_desc& D = pool->desc;
  if (Lc.window < 1 || Lc.window > BN + 1) {
    set_error("prefill: the narrow-window kernel needs 1 <= W <= %d", BN + 1);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  NParams p{};
  p.B = Lc.B;
  p.n_q = Lc.n_q;
  p.Hq = Lc.Hq;
  p.Hkv = Lc.Hkv;
  p.G = Lc.Hq / Lc.Hkv;
  p.window = Lc.window;
  p.start_pos = Lc.start_pos;
  p.seq_ids = Lc.seq_ids;
  p.ring_k = pool->ring_k;
  p.ring_v = pool->ring_v;
  p.ring_k8 = pool->ring_k8;
  p.ring_v8 = pool->ring_v8;
  p.fp8 = pool->fp8 ? 1 : 0;
  if (pool->fp8) {
    const int n_layers = D.n_swa_layers + D.n_full_layers;
    p.k_scale = pool->scales + (size_t)(0 * n_layers + Lc.layer) * D.n_kv_heads;
    p.v_scale = pool->scales + (size_t)(1 * n_layers + Lc.layer) * D.n_kv_heads;
  }
  p.ring_layer = Lc.ring_layer;
  p.n_swa = D.n_swa_layers;
  p.max_seqs = D.max_seqs;
  p.ring_tma = pool->ring_tma ? 1 : 0;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)Lc.d));
  p.n_tiles = (Lc.n_q + BM - 1) / BM;
  p.max_start = 0x7fffffffLL - Lc.n_q - 2 * BN;
  p.err = pool->err;
  if (Lc.n_q == 0 || Lc.B == 0) return HSWA_OK;
  const int64_t units = (int64_t)p.n_tiles * Lc.B * Lc.Hkv;
  if (units > 0x7fffffff) {
    set_error("prefill: too many work units");
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  p.n_units = (int)units;
  const int sms = pool->sms;
  const int grid = p.n_units < sms ? p.n_units : sms;

  const CUtensorMap& rk = pool->ring_tma ? pool->tm_ring_k : Lc.tm_k;
  const CUtensorMap& rv = pool->ring_tma ? pool->tm_ring_v : Lc.tm_v;
  if (Lc.d == 128) {
    const int smem = NLayout<128>::BYTES + 1024;
    cudaFuncSetAttribute(prefill_narrow_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_narrow_kernel<128><<<grid, NTHREADS, smem, stream>>>(p, Lc.tm_q, Lc.tm_k, Lc.tm_v, rk, rv, Lc.tm_o);
  } else {
    const int smem = NLayout<64>::BYTES + 1024;
    cudaFuncSetAttribute(prefill_narrow_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_narrow_kernel<64><<<grid, NTHREADS, smem, stream>>>(p, Lc.tm_q, Lc.tm_k, Lc.tm_v, rk, rv, Lc.tm_o);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("prefill: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

}  // namespace hswa

// prefill_narrow.cu -- causal sliding-window prefill for narrow windows (W <= 129), where the
// band of every 128-row query tile lies in at most two 128-key tiles.
//
// Math ("Sliding Window Attention (SWA) no riron to jisso", section "formal definition",
// eqs. (1)-(5)): query i attends keys j in [max(0, i - W + 1), i] with weights
// softmax_j(q_i . k_j / sqrt(d)) on v_j; query head h reads KV head h / G (section
// "Mistral: SWA and GQA"). Tiles outside the band are never loaded (section "sparsity:
// Flash Attention and BlockSparse").
//
// Work unit = (query tile t, batch row b, KV head g). The band of tile t covers key tiles
// t - 1 and t (relative to the chunk start; tile -1 is the rolling buffer). Both key tiles
// are loaded once per unit and stay in shared memory while the G query heads of KV head g
// stream through two slots: slot q takes heads g*G + q, g*G + q + 2, ...
//   warps 0-3 / 4-7  softmax + epilogue of slot 0 / slot 1 (one thread per TMEM lane)
//   warp 8           K/V producer (TMA for chunk rows and aligned ring tiles, cp.async for
//                    the others)
//   warp 9           MMA issuer for both slots in a fixed alternating order (one thread; the
//                    two softmax warpgroups then take turns with the tensor core); owns TMEM
//   warp 10          Q producer: the next head of a slot is loaded as soon as that slot's last
//                    S MMA of the current head has read its Q tile, so the load overlaps the
//                    slot's last softmax, P V and epilogue
//   warp 11          completes the warpgroup
// TMEM: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D); P is written over S.
// Shared memory: Q 2 tiles, K 2 tiles, V 2 tiles, output staging 2 x 16 KB.
#include "common.cuh"
#include "internal.h"
#include "prefill_tile.cuh"

namespace hswa {

namespace {

constexpr int NSLOT = 2;          // query-head slots
constexpr int NKT = 2;            // key tiles per unit (at most)
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
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NSLOT * TILE;
  static constexpr int V_OFF = K_OFF + NKT * TILE;
  static constexpr int O_OFF = V_OFF + NKT * TILE;  // 4 KB output staging per softmax warp
  static constexpr int BAR_OFF = O_OFF + 2 * BLOCK;
  static constexpr int BYTES = BAR_OFF + 256;
  static_assert(BYTES + 1024 <= 227 * 1024, "shared memory per CTA");
  static constexpr int O_COL0 = 256;
};

struct NBars {
  uint64_t q_full[NSLOT], q_empty[NSLOT];
  uint64_t kv_full[NKT], kv_empty[NKT];  // K and V of one key tile land together
  uint64_t s_full[NSLOT], p_full[NSLOT], o_full[NSLOT];
  uint32_t tmem_base;
};

struct NGeo {
  int t, b, g, P;
  int i0, i1;    // first / last valid absolute query position of the tile
  int jlo, nkt;  // first key tile (relative to the chunk start) and the number of key tiles
  int nh[NSLOT]; // heads of each slot
};

__device__ __forceinline__ int nwindow_lo(const NParams& p, int i) {
  const int lo = i - p.window + 1;
  return lo > 0 ? lo : 0;
}

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
  const int r0 = G.t * BM;
  const int r1 = (r0 + BM - 1 < p.n_q - 1) ? r0 + BM - 1 : p.n_q - 1;
  G.i0 = G.P + r0;
  G.i1 = G.P + r1;
  G.jlo = (int)floordiv(nwindow_lo(p, G.i0) - G.P, BN);
  G.nkt = (int)floordiv(G.i1 - G.P, BN) - G.jlo + 1;
  G.nh[0] = (p.G + 1) / 2;
  G.nh[1] = p.G / 2;
}

// ---------------------------------------------------------------- K/V producer

template <int D>
__device__ void kv_producer(const NParams& p, uint8_t* smem, NBars* bars, const CUtensorMap* tm_k,
                            const CUtensorMap* tm_v, const CUtensorMap* tm_rk, const CUtensorMap* tm_rv) {
  using L = NLayout<D>;
  const int lane = threadIdx.x & 31;
  uint32_t nkv[NKT] = {0, 0};  // loads per key-tile slot (kv_empty / kv_full phase)
  for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x) {
    NGeo G;
    make_ngeo(p, unit, G);
    const int seq = p.seq_ids ? p.seq_ids[G.b] : 0;
    const bool seq_ok = seq >= 0 && seq < p.max_seqs;
    const int64_t ring_row = seq_ok ? ((int64_t)seq * p.n_swa + p.ring_layer) * p.Hkv + G.g : 0;
    const bool ring_fast = p.ring_tma && (G.P % BN) == 0;
#pragma unroll
    for (int jj = 0; jj < NKT; ++jj) {
      if (jj >= G.nkt) break;
      const int j = G.jlo + jj;
      if (!mbar_wait(&bars->kv_empty[jj], (nkv[jj] & 1) ^ 1, p.err)) return;
      ++nkv[jj];
      uint8_t* dk = smem + L::K_OFF + jj * L::TILE;
      uint8_t* dv = smem + L::V_OFF + jj * L::TILE;
      if (j >= 0) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars->kv_full[jj], 2 * L::TILE);
          for (int dh = 0; dh < D / 64; ++dh) {
            tma_load_4d(dk + dh * L::BLOCK, tm_k, &bars->kv_full[jj], dh * 64, G.g, BN * j, G.b);
            tma_load_4d(dv + dh * L::BLOCK, tm_v, &bars->kv_full[jj], dh * 64, G.g, BN * j, G.b);
          }
        }
      } else if (ring_fast) {
        // W is a multiple of 128 and the chunk starts on a tile boundary: the tile is one box
        if (lane == 0) {
          if (!seq_ok) record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
          const int slot = (G.P + BN * j) % p.window;
          const int row = seq_ok ? (int)ring_row : -1;  // outside the map: zero fill
          mbar_arrive_expect_tx(&bars->kv_full[jj], 2 * L::TILE);
          for (int dh = 0; dh < D / 64; ++dh) {
            tma_load_3d(dk + dh * L::BLOCK, tm_rk, &bars->kv_full[jj], dh * 64, slot, row);
            tma_load_3d(dv + dh * L::BLOCK, tm_rv, &bars->kv_full[jj], dh * 64, slot, row);
          }
        }
      } else {
        if (!seq_ok && lane == 0) record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
        const int held_lo = (G.P - p.window > 0) ? G.P - p.window : 0;
        const int64_t base = ring_row * p.window * D;
        if (p.fp8) {
          ring_rows_fp8<D>(p.ring_k8 + base, seq_ok, held_lo, G.P, p.window, p.k_scale[G.g], dk, G.P + BN * j, lane);
          ring_rows_fp8<D>(p.ring_v8 + base, seq_ok, held_lo, G.P, p.window, p.v_scale[G.g], dv, G.P + BN * j, lane);
        } else {
          ring_rows_cpasync<D>(p.ring_k + base, seq_ok, held_lo, G.P, p.window, dk, G.P + BN * j, lane);
          ring_rows_cpasync<D>(p.ring_v + base, seq_ok, held_lo, G.P, p.window, dv, G.P + BN * j, lane);
        }
        if (lane == 0) mbar_arrive(&bars->kv_full[jj]);
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
        // the slot's Q buffer is free once its last S MMA of the previous head has completed
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

// One thread issues both slots' MMAs in a fixed alternating order, step by step (a step is one
// key tile of the slots' current heads): O_q += P_q V of the slot's previous S, then the slot's
// next S. While one slot's softmax runs, the tensor core works on the other slot's products.
template <int D>
__device__ void mma_issuer(const NParams& p, uint8_t* smem, NBars* bars, uint32_t tbase) {
  using L = NLayout<D>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
  const uint32_t q_base = smem_u32(smem + L::Q_OFF);
  const uint32_t k_base = smem_u32(smem + L::K_OFF);
  const uint32_t v_base = smem_u32(smem + L::V_OFF);
  uint32_t np = 0;    // bit q: p_full phase of slot q
  uint32_t nqf = 0;   // bit q: q_full phase of slot q
  uint32_t kvph = 0;  // bit jj: kv_full phase of key-tile slot jj

  for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x) {
    NGeo G;
    make_ngeo(p, unit, G);
    uint32_t kv_ready = 0;  // bit jj: key tile jj of this unit has landed
    int pend_jj[NSLOT] = {-1, -1};  // key tile of a slot's S whose P V is not issued yet
    bool pend_last[NSLOT] = {false, false};  // ... and it is the head's last key tile
    auto drain = [&](int q) -> bool {
      if (pend_jj[q] < 0) return true;
      if (!mbar_wait(&bars->p_full[q], (np >> q) & 1u, p.err)) return false;
      np ^= 1u << q;
      tc_fence_after();
      const int jj = pend_jj[q];
      const uint32_t vb = v_base + jj * L::TILE;
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        const uint64_t bdesc = smem_desc_sw128(vb + kk * 16 * 128, L::BLOCK, 1024);
        umma_ts(tbase + L::O_COL0 + q * 128, tbase + q * 128 + kk * 8, bdesc, IDESC_PV,
                (jj > 0 || kk > 0) ? 1u : 0u);
      }
      if (pend_last[q]) umma_commit(&bars->o_full[q]);
      pend_jj[q] = -1;
      return true;
    };
    const int nk = G.nh[0] > G.nh[1] ? G.nh[0] : G.nh[1];
    for (int k = 0; k < nk; ++k) {
      for (int jj = 0; jj < G.nkt; ++jj) {
        if (!((kv_ready >> jj) & 1u)) {
          if (!mbar_wait(&bars->kv_full[jj], (kvph >> jj) & 1u, p.err)) return;
          tc_fence_after();
          kv_ready |= 1u << jj;
        }
#pragma unroll
        for (int q = 0; q < NSLOT; ++q) {
          // P of the slot's previous key tile lives in its S columns: that P V goes first
          if (!drain(q)) return;
          if (k >= G.nh[q]) continue;
          if (jj == 0) {  // a new head of the slot: its Q tile
            if (!mbar_wait(&bars->q_full[q], (nqf >> q) & 1u, p.err)) return;
            nqf ^= 1u << q;
            tc_fence_after();
          }
          const uint32_t qb = q_base + q * L::TILE, kb = k_base + jj * L::TILE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::BLOCK + (kk & 3) * 32;
            umma_ss(tbase + q * 128, smem_desc_sw128(qb + off, 16, 1024), smem_desc_sw128(kb + off, 16, 1024),
                    IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars->s_full[q]);
          if (jj == G.nkt - 1) umma_commit(&bars->q_empty[q]);  // this head's Q tile is read
          pend_jj[q] = jj;
          pend_last[q] = jj == G.nkt - 1;
        }
        // the last products on key tile jj - 1 have just been issued: the producer may refill it
        // for the next unit while this step's work runs
        if (k == nk - 1 && jj > 0) {
          umma_commit(&bars->kv_empty[jj - 1]);
          kvph ^= 1u << (jj - 1);
        }
      }
    }
    // the last products read the unit's last V tile: issue them, then release that tile
#pragma unroll
    for (int q = 0; q < NSLOT; ++q)
      if (!drain(q)) return;
    umma_commit(&bars->kv_empty[G.nkt - 1]);
    kvph ^= 1u << (G.nkt - 1);
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
  const uint32_t s_col = q * 128;
  const uint32_t o_col = L::O_COL0 + q * 128;
  const float sl2 = p.scale_log2;
  uint8_t* stage = smem + L::O_OFF + q * L::BLOCK + wq * 4096;
  uint32_t ns = 0;  // S tiles consumed (s_full phase)
  uint32_t no = 0;  // heads finished (o_full phase)

  for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x) {
    NGeo G;
    make_ngeo(p, unit, G);
    const int lo_last = nwindow_lo(p, G.i1);
    // W = 128 and no row's band clipped at the sequence start: the rotated-chunk mask applies
    const bool w128 = p.window == 128 && G.nkt == 2 && G.i0 >= 127 && G.jlo == G.t - 1;
    const int i = G.i0 + r;
    const int lo_i = nwindow_lo(p, i);
    for (int k = 0; k < G.nh[q]; ++k) {
      float m_used = -INFINITY;
      float l = 0.f;
      for (int jj = 0; jj < G.nkt; ++jj) {
        if (!mbar_wait(&bars->s_full[q], ns & 1, p.err)) return;
        ++ns;
        tc_fence_after();
        // columns of this row inside the band: [c_lo, c_hi] (edge tiles only)
        const int kb = G.P + BN * (G.jlo + jj);
        const bool edge = !(kb + BN - 1 <= G.i0 && kb >= lo_last);
        if (w128)
          softmax_tile<D, 2>(trow, s_col, o_col, sl2, true, 0, 0, m_used, l, jj > 0, wq, jj == 0);
        else
          softmax_tile<D, 0>(trow, s_col, o_col, sl2, edge, lo_i - kb, i - kb, m_used, l, jj > 0);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[q]);
      }
      if (!mbar_wait(&bars->o_full[q], no & 1, p.err)) return;
      ++no;
      tc_fence_after();
      store_output<D>(trow, o_col, l, stage, lane, tm_o, G.g * p.G + q + 2 * k, G.t * BM + wq * 32, G.b, p.n_q);
      // O of this head has been read: the next head's first P V may overwrite it (ordered by
      // this warpgroup's next p_full arrival)
      tc_fence_before();
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
    }
    for (int jj = 0; jj < NKT; ++jj) {
      mbar_init(&bars->kv_full[jj], 1);
      mbar_init(&bars->kv_empty[jj], 1);
    }
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

// prefill_sm100.cu -- causal sliding-window and full causal attention for one chunk,
// on Blackwell tensor cores (tcgen05 + TMEM, operands staged by TMA).
//
// Math ("Sliding Window Attention (SWA) no riron to jisso", section "formal
// definition", eqs. (1)-(5)): query i attends keys j in [lo(i), i] with
// lo(i) = max(0, i - W + 1) (W = 0: lo = 0, full causal), weights
// softmax_j(q_i . k_j / sqrt(d)) on v_j. Query head h reads KV head h / G (GQA,
// section "Mistral: SWA and GQA"). Tiles of the (query, key) plane that lie wholly
// outside the band are never loaded or multiplied (section "sparsity: Flash
// Attention and BlockSparse": blocks outside the window are skipped); only tiles
// that the band edge crosses are masked.
//
// CTA = 2 query tiles of 128 rows (one batch row b, one query head h).
//   warp 0      producer: Q once, then K/V tiles into a 2-stage ring of shared-memory
//               buffers (TMA for chunk rows and pages; cp.async for rolling-buffer
//               rows that are not 128-aligned).
//   warp 1      MMA issuer (one thread): S_q = Q_q K_j^T into TMEM, O_q += P_q V_j
//               with P_q read from TMEM; also allocates/frees TMEM.
//   warps 4-7   softmax for query tile 0, warps 8-11 for query tile 1: one thread per
//               row (TMEM lane), online max/sum in the exp2 domain with lazy O
//               rescaling, P written back over S as packed bf16, and the epilogue.
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D).
//
// Key tiles. Sliding-window layers: tile j covers positions [P + 128 j, P + 128 j + 128)
// with P the chunk's first position, so tiles j >= 0 are rows of the chunk input and
// tiles j < 0 are rolling-buffer slots (pos mod W). Full layers: tile j covers
// absolute positions [128 j, 128 j + 128) = two 64-token pages.
#include "common.cuh"
#include "internal.h"

namespace hswa {

namespace {

constexpr int BM = 128;     // query rows per tile
constexpr int BN = 128;     // keys per tile
constexpr int NQT = 2;      // query tiles per CTA
constexpr int NSTAGE = 2;   // K/V pipeline depth
constexpr int NTHREADS = 384;
constexpr float kTau = 8.0f;  // lazy rescale threshold (log2 units): P stays <= 2^8

struct Params {
  int B, n_q, Hq, Hkv, G;
  int window;   // W >= 1, or 0 for full causal
  int is_full;
  const int64_t* start_pos;
  const int32_t* seq_ids;
  const int32_t* page_table;
  int pt_stride;
  uint16_t* o;
  const uint16_t* ring_k;
  const uint16_t* ring_v;
  int ring_layer, n_swa, max_seqs, ring_tma;
  int full_layer;
  int64_t pages;
  float scale_log2;
  int n_pairs;
  int* err;
};

template <int D>
struct Layout {
  static constexpr int BLOCK = BM * 128;           // one [128 rows][64 elems] swizzled block = 16 KB
  static constexpr int TILE = BLOCK * (D / 64);    // one 128 x D tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NQT * TILE;
  static constexpr int V_OFF = K_OFF + NSTAGE * TILE;
  static constexpr int BAR_OFF = V_OFF + NSTAGE * TILE;
  static constexpr int BYTES = BAR_OFF + 256;
  static constexpr int O_COL0 = 256;
  static constexpr int O_STRIDE = 128;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NSTAGE], k_empty[NSTAGE], v_full[NSTAGE], v_empty[NSTAGE];
  uint64_t s_full[NQT], p_full[NQT], o_full[NQT];
  uint64_t v_fix;  // TMA completion of the page tile that holds the last key (before its tail is zeroed)
  uint32_t tmem_base;
};

// Geometry of one CTA's work, computed identically by every role.
struct Geo {
  int b, h, g;
  int64_t P;             // absolute position of the chunk's first row
  int t[NQT];            // query tile index within the chunk
  bool act[NQT];
  int64_t i0[NQT], i1[NQT];  // first / last valid absolute query position of each tile
  int64_t jlo[NQT], jhi[NQT];
  int64_t jb, je;        // union of needed key tiles, inclusive
};

__device__ __forceinline__ int64_t window_lo(const Params& p, int64_t i) {
  if (p.window <= 0) return 0;
  const int64_t lo = i - p.window + 1;
  return lo > 0 ? lo : 0;
}

__device__ __forceinline__ int64_t key_base(const Params& p, const Geo& G, int64_t j) {
  return p.is_full ? (int64_t)BN * j : G.P + (int64_t)BN * j;
}

__device__ __forceinline__ void make_geo(const Params& p, Geo& G) {
  G.h = blockIdx.x;
  const int pair = p.n_pairs - 1 - (int)blockIdx.y;  // longest causal work first
  G.b = blockIdx.z;
  G.g = G.h / p.G;
  G.P = p.start_pos ? p.start_pos[G.b] : 0;
  G.jb = INT64_MAX;
  G.je = INT64_MIN;
  for (int q = 0; q < NQT; ++q) {
    G.t[q] = pair * NQT + q;
    const int64_t r0 = (int64_t)G.t[q] * BM;
    G.act[q] = r0 < p.n_q;
    if (!G.act[q]) continue;
    const int64_t r1 = (r0 + BM - 1 < p.n_q - 1) ? r0 + BM - 1 : p.n_q - 1;
    G.i0[q] = G.P + r0;
    G.i1[q] = G.P + r1;
    if (p.is_full) {
      G.jlo[q] = 0;
      G.jhi[q] = floordiv(G.i1[q], BN);
    } else {
      G.jlo[q] = floordiv(window_lo(p, G.i0[q]) - G.P, BN);
      G.jhi[q] = floordiv(G.i1[q] - G.P, BN);
    }
    if (G.jlo[q] < G.jb) G.jb = G.jlo[q];
    if (G.jhi[q] > G.je) G.je = G.jhi[q];
  }
}

__device__ __forceinline__ bool needs(const Geo& G, int q, int64_t j) {
  return G.act[q] && j >= G.jlo[q] && j <= G.jhi[q];
}

// All (row, key) pairs of the tile are inside the band.
__device__ __forceinline__ bool mask_free(const Params& p, const Geo& G, int q, int64_t j) {
  const int64_t kb = key_base(p, G, j);
  return kb + BN - 1 <= G.i0[q] && kb >= window_lo(p, G.i1[q]);
}

// ---------------------------------------------------------------- producer

// Rolling-buffer rows of one key tile with cp.async (general W and chunk start):
// rows whose position is not held by the ring (or is negative) are zero-filled.
template <int D>
__device__ __forceinline__ void ring_tile_cpasync(const Params& p, const Geo& G, const uint16_t* ring,
                                                  uint8_t* dst, int64_t kb, int lane) {
  const int seq = p.seq_ids ? p.seq_ids[G.b] : 0;
  const bool seq_ok = seq >= 0 && seq < p.max_seqs;
  if (!seq_ok && lane == 0) record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
  const int64_t row_base = seq_ok ? (((int64_t)seq * p.n_swa + p.ring_layer) * p.Hkv + G.g) * p.window : 0;
  const int64_t held_lo = (G.P - p.window > 0) ? G.P - p.window : 0;
  const uint32_t sdst = smem_u32(dst);
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int idx = lane; idx < BN * CH; idx += 32) {
    const int r = idx / CH;
    const int c = idx % CH;
    const int64_t pos = kb + r;
    const bool held = seq_ok && pos >= held_lo && pos < G.P;
    const uint16_t* src = ring + (held ? (row_base + (pos % p.window)) * D + c * 8 : 0);
    const int blk = c >> 3, cc = c & 7;
    const uint32_t off = blk * (BM * 128) + r * 128 + ((cc ^ (r & 7)) << 4);
    cp_async_16(sdst + off, src, held ? 16u : 0u);
  }
  cp_async_wait_all();
  fence_proxy_async_smem();
  __syncwarp();
}

template <int D>
__device__ void producer(const Params& p, const Geo& G, uint8_t* smem, Bars* bars, const CUtensorMap* tm_q,
                         const CUtensorMap* tm_k, const CUtensorMap* tm_v, const CUtensorMap* tm_rk,
                         const CUtensorMap* tm_rv) {
  using L = Layout<D>;
  const int lane = threadIdx.x & 31;
  if (lane == 0) {
    int nact = 0;
    for (int q = 0; q < NQT; ++q) nact += G.act[q];
    mbar_arrive_expect_tx(&bars->q_full, nact * L::TILE);
    for (int q = 0; q < NQT; ++q) {
      if (!G.act[q]) continue;
      for (int dh = 0; dh < D / 64; ++dh)
        tma_load_4d(smem + L::Q_OFF + q * L::TILE + dh * L::BLOCK, tm_q, &bars->q_full, dh * 64, G.h,
                    G.t[q] * BM, G.b);
    }
  }
  // highest key position any query of this CTA may need
  int64_t kmax = 0;
  for (int q = 0; q < NQT; ++q)
    if (G.act[q] && G.i1[q] > kmax) kmax = G.i1[q];
  const int seq = (!p.is_full && p.seq_ids) ? p.seq_ids[G.b] : 0;
  const bool ring_fast = p.ring_tma && (G.P % BN) == 0;

  int it = 0;
  for (int64_t j = G.jb; j <= G.je; ++j, ++it) {
    const int s = it % NSTAGE;
    const uint32_t ph = (it / NSTAGE) & 1;
    const int64_t kb = key_base(p, G, j);
    for (int kv = 0; kv < 2; ++kv) {
      uint64_t* full = kv ? &bars->v_full[s] : &bars->k_full[s];
      uint64_t* empty = kv ? &bars->v_empty[s] : &bars->k_empty[s];
      uint8_t* dst = smem + (kv ? L::V_OFF : L::K_OFF) + s * L::TILE;
      if (!mbar_wait(empty, ph ^ 1, p.err)) return;
      if (p.is_full) {
        // Rows of the last page past the last key hold stale memory; P is 0 there, but
        // 0 * NaN would still poison P V, so that V tile is zeroed past kmax before use.
        const bool fix = kv == 1 && kb <= kmax && kmax < kb + BN - 1 && ((kmax + 1) % 64) != 0;
        uint64_t* land = fix ? &bars->v_fix : full;
        if (lane == 0) {
          mbar_arrive_expect_tx(land, L::TILE);
          const CUtensorMap* tm = kv ? tm_v : tm_k;
          for (int half = 0; half < 2; ++half) {
            const int64_t pos0 = kb + 64 * half;
            const int64_t lp = pos0 / 64;
            int64_t row = -1;  // outside the map: zero fill
            if (pos0 <= kmax) {
              int32_t page = -1;
              if (lp < p.pt_stride) page = p.page_table[(int64_t)G.b * p.pt_stride + lp];
              if (page < 0 || page >= p.pages) {
                record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
              } else {
                row = ((int64_t)p.full_layer * p.pages + page) * p.Hkv + G.g;
              }
            }
            for (int dh = 0; dh < D / 64; ++dh)
              tma_load_3d(dst + dh * L::BLOCK + half * 64 * 128, tm, land, dh * 64, 0, (int)row);
          }
        }
        if (fix) {
          __syncwarp();
          if (!mbar_wait(&bars->v_fix, 0, p.err)) return;
          const int r0 = (int)(kmax - kb + 1);
          for (int idx = lane; idx < (BN - r0) * (D / 8); idx += 32) {
            const int r = r0 + idx / (D / 8);
            const int c = idx % (D / 8);
            *reinterpret_cast<uint4*>(dst + (c >> 3) * L::BLOCK + r * 128 + (c & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(full);
        }
      } else if (j >= 0) {
        if (lane == 0) {
          mbar_arrive_expect_tx(full, L::TILE);
          const CUtensorMap* tm = kv ? tm_v : tm_k;
          for (int dh = 0; dh < D / 64; ++dh)
            tma_load_4d(dst + dh * L::BLOCK, tm, full, dh * 64, G.g, (int)(BN * j), G.b);
        }
      } else if (ring_fast) {
        if (lane == 0) {
          mbar_arrive_expect_tx(full, L::TILE);
          const CUtensorMap* tm = kv ? tm_rv : tm_rk;
          const int slot = (int)(kb % p.window);
          int row = -1;  // outside the map: zero fill
          if (seq >= 0 && seq < p.max_seqs)
            row = (int)(((int64_t)seq * p.n_swa + p.ring_layer) * p.Hkv + G.g);
          else
            record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
          for (int dh = 0; dh < D / 64; ++dh) tma_load_3d(dst + dh * L::BLOCK, tm, full, dh * 64, slot, row);
        }
      } else {
        ring_tile_cpasync<D>(p, G, kv ? p.ring_v : p.ring_k, dst, kb, lane);
        if (lane == 0) mbar_arrive(full);
      }
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------- MMA issuer

template <int D>
__device__ void mma_issuer(const Params& p, const Geo& G, uint8_t* smem, Bars* bars, uint32_t tbase) {
  using L = Layout<D>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
  const uint32_t q_base = smem_u32(smem + L::Q_OFF);
  const uint32_t k_base = smem_u32(smem + L::K_OFF);
  const uint32_t v_base = smem_u32(smem + L::V_OFF);

  if (!mbar_wait(&bars->q_full, 0, p.err)) return;
  tc_fence_after();

  bool pend[NQT] = {false, false};
  bool started[NQT] = {false, false};
  uint32_t np[NQT] = {0, 0};
  int prev_s = 0;
  uint32_t prev_ph = 0;
  int it = 0;

  auto issue_pv = [&](int q, int s) {
    const uint32_t d_tmem = tbase + L::O_COL0 + q * L::O_STRIDE;
    const uint32_t a_tmem = tbase + q * 128;
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
      const uint64_t bdesc = smem_desc_sw128(v_base + s * L::TILE + kk * 16 * 128, L::BLOCK, 1024);
      umma_ts(d_tmem, a_tmem + kk * 8, bdesc, IDESC_PV, (started[q] || kk > 0) ? 1u : 0u);
    }
    started[q] = true;
  };

  for (int64_t j = G.jb; j <= G.je; ++j, ++it) {
    const int s = it % NSTAGE;
    const uint32_t ph = (it / NSTAGE) & 1;
    if (!mbar_wait(&bars->k_full[s], ph, p.err)) return;
    tc_fence_after();
    bool v_ready = false;
    for (int q = 0; q < NQT; ++q) {
      if (pend[q]) {
        if (!mbar_wait(&bars->p_full[q], np[q] & 1, p.err)) return;
        ++np[q];
        tc_fence_after();
        if (!v_ready) {
          if (!mbar_wait(&bars->v_full[prev_s], prev_ph, p.err)) return;
          tc_fence_after();
          v_ready = true;
        }
        issue_pv(q, prev_s);
        pend[q] = false;
      }
      if (needs(G, q, j)) {
        const uint32_t d_tmem = tbase + q * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::BLOCK + (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(q_base + q * L::TILE + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(k_base + s * L::TILE + off, 16, 1024);
          umma_ss(d_tmem, adesc, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[q]);
        pend[q] = true;
      }
    }
    umma_commit(&bars->k_empty[s]);
    if (it > 0) {
      if (!v_ready) {
        if (!mbar_wait(&bars->v_full[prev_s], prev_ph, p.err)) return;
        tc_fence_after();
      }
      umma_commit(&bars->v_empty[prev_s]);
    }
    prev_s = s;
    prev_ph = ph;
  }
  // drain the last tile's P V products
  bool v_ready = false;
  for (int q = 0; q < NQT; ++q) {
    if (!pend[q]) continue;
    if (!mbar_wait(&bars->p_full[q], np[q] & 1, p.err)) return;
    ++np[q];
    tc_fence_after();
    if (!v_ready) {
      if (!mbar_wait(&bars->v_full[prev_s], prev_ph, p.err)) return;
      tc_fence_after();
      v_ready = true;
    }
    issue_pv(q, prev_s);
  }
  for (int q = 0; q < NQT; ++q)
    if (G.act[q]) umma_commit(&bars->o_full[q]);
}

// ---------------------------------------------------------------- softmax + epilogue

template <int D>
__device__ void softmax_wg(const Params& p, const Geo& G, Bars* bars, uint32_t tbase, int q) {
  using L = Layout<D>;
  if (!G.act[q]) return;
  const int wq = (threadIdx.x >> 5) & 3;
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;
  const int64_t i = G.i0[q] + r;
  const int64_t lo_i = window_lo(p, i);
  const uint32_t trow = tbase + ((uint32_t)(wq * 32) << 16);
  const uint32_t s_col = q * 128;
  const uint32_t o_col = L::O_COL0 + q * L::O_STRIDE;
  const float sl2 = p.scale_log2;

  float m_used = -INFINITY;
  float l = 0.f;
  uint32_t n_done = 0;

  for (int64_t j = G.jlo[q]; j <= G.jhi[q]; ++j) {
    if (!mbar_wait(&bars->s_full[q], n_done & 1, p.err)) return;
    tc_fence_after();
    const int64_t kb = key_base(p, G, j);
    const bool full_tile = mask_free(p, G, q, j);
    // column range of this row inside the band
    const int64_t c_lo = lo_i - kb;
    const int64_t c_hi = i - kb;

    float mx = -INFINITY;
#pragma unroll
    for (int c0 = 0; c0 < BN; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(trow + s_col + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        float sv = __uint_as_float(v[k]);
        if (!full_tile && (c0 + k < c_lo || c0 + k > c_hi)) sv = -INFINITY;
        mx = fmaxf(mx, sv);
      }
    }
    const float m_tile = mx * sl2;
    float alpha = 1.f;
    bool resc = false;
    if (m_tile > m_used + kTau) {
      if (m_used != -INFINITY) {
        alpha = ex2_approx(m_used - m_tile);
        resc = true;
      }
      l *= alpha;
      m_used = m_tile;
    }
    if (__any_sync(0xffffffffu, resc) && n_done > 0) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(trow + o_col + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
        tmem_st32(trow + o_col + c0, v);
      }
      tmem_wait_st();
    }
    const float moff = (m_used == -INFINITY) ? 0.f : m_used;
#pragma unroll
    for (int c0 = 0; c0 < BN; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(trow + s_col + c0, v);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        float s0 = __uint_as_float(v[k]);
        float s1 = __uint_as_float(v[k + 1]);
        if (!full_tile) {
          if (c0 + k < c_lo || c0 + k > c_hi) s0 = -INFINITY;
          if (c0 + k + 1 < c_lo || c0 + k + 1 > c_hi) s1 = -INFINITY;
        }
        const float p0 = ex2_approx(fmaf(s0, sl2, -moff));
        const float p1 = ex2_approx(fmaf(s1, sl2, -moff));
        l += p0 + p1;
        pk[k >> 1] = pack_bf16x2(p0, p1);
      }
      tmem_st16(trow + s_col + (c0 >> 1), pk);
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bars->p_full[q]);
    ++n_done;
  }

  if (n_done == 0) return;
  if (!mbar_wait(&bars->o_full[q], 0, p.err)) return;
  tc_fence_after();
  const int64_t row = (int64_t)G.t[q] * BM + r;
  const bool valid = row < p.n_q;
  const float inv = 1.f / l;
  uint16_t* out = p.o + (((int64_t)G.b * p.n_q + row) * p.Hq + G.h) * D;
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(trow + o_col + c0, v);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int k = 0; k < 32; k += 2)
      pk[k >> 1] = pack_bf16x2(__uint_as_float(v[k]) * inv, __uint_as_float(v[k + 1]) * inv);
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(out + c0);
#pragma unroll
      for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_rk, const __grid_constant__ CUtensorMap tm_rv) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::BAR_OFF);
  const int warp = threadIdx.x >> 5;

  if (read_error(p.err) != 0) return;  // a pending device error: skip the work

  Geo G;
  make_geo(p, G);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int q = 0; q < NQT; ++q) {
      mbar_init(&bars->s_full[q], 1);
      mbar_init(&bars->p_full[q], 128);
      mbar_init(&bars->o_full[q], 1);
    }
    mbar_init(&bars->v_fix, 1);
    fence_barrier_init();
  }
  if (warp == 0 && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;

  if (warp == 0) {
    producer<D>(p, G, smem, bars, &tm_q, &tm_k, &tm_v, &tm_rk, &tm_rv);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) mma_issuer<D>(p, G, smem, bars, tbase);
    __syncwarp();
  } else if (warp >= 4) {
    softmax_wg<D>(p, G, bars, tbase, (warp - 4) >> 2);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace

int launch_prefill(const PrefillLaunch& Lc, cudaStream_t stream) {
  const hswa_pool* pool = Lc.pool;
  const hswa_pool_desc& D = pool->desc;
  Params p{};
  p.B = Lc.B;
  p.n_q = Lc.n_q;
  p.Hq = Lc.Hq;
  p.Hkv = Lc.Hkv;
  p.G = Lc.Hq / Lc.Hkv;
  p.window = Lc.window;
  p.is_full = Lc.window == 0;
  p.start_pos = Lc.start_pos;
  p.seq_ids = Lc.seq_ids;
  p.page_table = Lc.page_table;
  p.pt_stride = Lc.pt_stride;
  p.o = Lc.o;
  p.ring_k = pool->ring_k;
  p.ring_v = pool->ring_v;
  p.ring_layer = Lc.ring_layer;
  p.n_swa = D.n_swa_layers;
  p.max_seqs = D.max_seqs;
  p.ring_tma = pool->ring_tma ? 1 : 0;
  p.full_layer = Lc.full_layer;
  p.pages = D.pages_per_full_layer;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)Lc.d));
  p.n_pairs = (int)((Lc.n_q + BM * NQT - 1) / (BM * NQT));
  p.err = pool->err;
  if (Lc.n_q == 0 || Lc.B == 0) return HSWA_OK;

  const dim3 grid(Lc.Hq, p.n_pairs, Lc.B);
  const CUtensorMap& rk = pool->ring_tma ? pool->tm_ring_k : Lc.tm_k;
  const CUtensorMap& rv = pool->ring_tma ? pool->tm_ring_v : Lc.tm_v;
  cudaError_t e;
  if (Lc.d == 128) {
    const int smem = Layout<128>::BYTES + 1024;
    cudaFuncSetAttribute(prefill_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_kernel<128><<<grid, NTHREADS, smem, stream>>>(p, Lc.tm_q, Lc.tm_k, Lc.tm_v, rk, rv);
  } else {
    const int smem = Layout<64>::BYTES + 1024;
    cudaFuncSetAttribute(prefill_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_kernel<64><<<grid, NTHREADS, smem, stream>>>(p, Lc.tm_q, Lc.tm_k, Lc.tm_v, rk, rv);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("prefill: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

}  // namespace hswa

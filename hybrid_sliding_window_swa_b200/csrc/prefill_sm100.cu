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
// This kernel serves full layers and sliding windows W > 129; narrower windows go to
// prefill_narrow.cu (launch_prefill dispatches). The per-row softmax step and the output
// epilogue are shared with it (prefill_tile.cuh).
//
// Work unit: two 128-row query tiles that share every key tile. With an even number G of query
// heads per KV head the two tiles are the same rows of two heads of one GQA group (unit = query
// tile, batch row, KV head, head pair): they need the same key tiles, so each K/V tile loaded into
// shared memory feeds both and the two slots' work is equal. With odd G the unit is two
// consecutive query tiles of one head. The grid is persistent (one CTA per SM) and walks the
// units in static rounds (serpentine: every other round from the last CTA down), in blocks of query tiles (latest first) inside which the units
// of one (batch row, KV head) are consecutive, so the CTAs share that group's K/V tiles in L2.
//   warps 0-3   softmax for slot 0, warps 4-7 for slot 1: one thread per
//               row (TMEM lane); all 128 scores of a row in registers, online max/sum
//               in the exp2 domain with lazy O rescaling, MUFU exponentials (an FMA-pipe
//               polynomial can take a share, HSWA_POLY_PER8), P written back over S as
//               packed bf16, and the epilogue (O / l -> bf16, staged in shared memory per
//               warp and written by TMA stores).
//   warps 8-11  a third warpgroup that gives its registers to the softmax warpgroups
//               (setmaxnreg, by default 2 x 128 x 216 + 128 x 72 = the 384 x 168 the CTA launches with):
//   warp 8      producer: Q of each unit, then K/V tiles into a 2-stage ring of
//               shared-memory buffers (TMA for chunk rows, aligned ring tiles and
//               pages; cp.async for rolling-buffer rows that are not 128-aligned).
//   warp 9      MMA issuer (one thread): S_q = Q_q K_j^T into TMEM, O_q += P_q V_j
//               with P_q read from TMEM; also allocates/frees TMEM.
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D).
//
// Key tiles. Sliding-window layers: tile j covers positions [P + 128 j, P + 128 j + 128)
// with P the chunk's first position, so tiles j >= 0 are rows of the chunk input and
// tiles j < 0 are rolling-buffer slots (pos mod W). Full layers: tile j covers
// absolute positions [128 j, 128 j + 128) = two 64-token pages.
#include "common.cuh"
#include "internal.h"
#include "prefill_tile.cuh"

namespace hswa {

namespace {

constexpr int NQT = 2;      // query tiles per unit
constexpr int NSTAGE = 2;   // K/V pipeline depth
constexpr int NWARPS = 12;         // 3 warpgroups: registers are granted per warpgroup
constexpr int NTHREADS = NWARPS * 32;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;

struct Params {
  int B, n_q, Hq, Hkv, G;
  int window;   // W >= 1, or 0 for full causal
  int is_full;
  const int64_t* start_pos;
  const int32_t* seq_ids;
  const int32_t* page_table;
  int pt_stride;
  const uint16_t* ring_k;
  const uint16_t* ring_v;
  const uint8_t* ring_k8;  // FP8 pools: the rings as E4M3 codes, and this layer's per-KV-head scales
  const uint8_t* ring_v8;
  const float* k_scale;
  const float* v_scale;
  int fp8;
  int conv;  // FP8 pages (full layer): page tiles are converted to bf16 in shared memory by warps 10-11
  int ring_layer, n_swa, max_seqs, ring_tma;
  int full_layer;
  int64_t pages;
  float scale_log2;
  int n_pairs;     // pairs of query tiles per (batch row, head)   (G odd)
  int n_tiles;     // query tiles per batch row                    (G even)
  int head_pairs;  // 1: a unit is one query tile of two heads of a GQA group
  int t_block;     // unit order: query tiles (or tile pairs) per block, see unit_order
  int n_units;
  int64_t max_start;  // largest start position that keeps every position below 2^31
  int* err;
};

template <int D>
struct Layout {
  static constexpr int BLOCK = BM * 128;           // one [128 rows][64 elems] swizzled block = 16 KB
  static constexpr int TILE = BLOCK * (D / 64);    // one 128 x D tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NQT * TILE;
  static constexpr int V_OFF = K_OFF + NSTAGE * TILE;
  static constexpr int O_OFF = V_OFF + NSTAGE * TILE;   // output staging: 4 KB (32 rows x 128 B) per softmax warp
  static constexpr int BAR_OFF = O_OFF + 2 * BLOCK;
  static constexpr int BYTES = BAR_OFF + 256;
  static_assert(BYTES + 1024 <= 227 * 1024, "shared memory per CTA");
  static constexpr int O_COL0 = 256;
  static constexpr int O_STRIDE = 128;
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[NSTAGE], k_empty[NSTAGE], v_full[NSTAGE], v_empty[NSTAGE];
  uint64_t raw_k[NSTAGE], raw_v[NSTAGE];  // FP8 page tiles landed (before conversion)
  uint64_t s_full[NQT], p_full[NQT], o_full[NQT];
  uint64_t v_fix;  // TMA completion of the page tile that holds the last key (before its tail is zeroed)
  uint32_t tmem_base;
};

// Geometry of one work unit, computed identically by every role.
// Positions are below 2^31 (checked on the host against start_pos bounds on the device).
struct Geo {
  int b, g;
  int hq[NQT];           // query head of each slot
  int P;                 // absolute position of the chunk's first row
  int t[NQT];            // query tile index within the chunk
  bool act[NQT];
  int i0[NQT], i1[NQT];  // first / last valid absolute query position of each tile
  int jlo[NQT], jhi[NQT];
  int jb, je;            // union of needed key tiles, inclusive
};

__device__ __forceinline__ int window_lo(const Params& p, int i) {
  if (p.window <= 0) return 0;
  const int lo = i - p.window + 1;
  return lo > 0 ? lo : 0;
}

__device__ __forceinline__ int key_base(const Params& p, const Geo& G, int j) {
  return p.is_full ? BN * j : G.P + BN * j;
}

// Unit order: query tiles (pairs of tiles for odd G) are cut into blocks of t_block, latest
// (longest causal) block first; inside a block the units of one (batch row, KV head) are
// consecutive, latest tile first. t_block = 1 is a plain latest-tile-first order (even tail); a
// block as long as the chunk makes all CTAs walk one group's key window together (its K/V tiles
// stay in L2 while Q and O stream through).
__device__ __forceinline__ void unit_order(int unit, int n_t, int n_bg, int n_in, int t_block, int& t,
                                           int& bg, int& in) {
  const int per_block = t_block * n_bg * n_in;
  const int k = unit / per_block;
  const int rem = unit - k * per_block;
  const int len = min(t_block, n_t - k * t_block);  // only the last block is shorter
  bg = rem / (len * n_in);
  const int r2 = rem - bg * (len * n_in);
  t = n_t - 1 - k * t_block - r2 / n_in;
  in = r2 - (r2 / n_in) * n_in;
}

// The unit a CTA takes in round r of the persistent loop: rounds go through the units in order,
// every other round from the last CTA down (serpentine), so with units sorted heaviest first each
// CTA's total work is nearly equal.
__device__ __forceinline__ int cta_unit(int r) {
  const int c = (HSWA_UNIT_SERPENTINE && (r & 1)) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x;
  return r * (int)gridDim.x + c;
}

__device__ __forceinline__ void make_geo(const Params& p, int unit, Geo& G) {
  int tq[NQT];
  int t, bg, in;
  if (p.head_pairs) {
    unit_order(unit, p.n_tiles, p.B * p.Hkv, p.G >> 1, p.t_block, t, bg, in);
    G.b = bg / p.Hkv;
    G.g = bg - G.b * p.Hkv;
#pragma unroll
    for (int q = 0; q < NQT; ++q) {
      tq[q] = t;
      G.hq[q] = G.g * p.G + 2 * in + q;
    }
  } else {
    unit_order(unit, p.n_pairs, p.B * p.Hkv, p.G, p.t_block, t, bg, in);
    G.b = bg / p.Hkv;
    G.g = bg - G.b * p.Hkv;
#pragma unroll
    for (int q = 0; q < NQT; ++q) {
      tq[q] = t * NQT + q;
      G.hq[q] = G.g * p.G + in;
    }
  }
  int64_t P = p.start_pos ? p.start_pos[G.b] : 0;
  if (P < 0 || P > p.max_start) {  // positions must stay below 2^31
    record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
    P = 0;
  }
  G.P = (int)P;
  G.jb = INT32_MAX;
  G.je = INT32_MIN;
#pragma unroll
  for (int q = 0; q < NQT; ++q) {
    G.t[q] = tq[q];
    const int r0 = G.t[q] * BM;
    G.act[q] = r0 < p.n_q;
    G.i0[q] = G.i1[q] = G.jlo[q] = 0;
    G.jhi[q] = -1;
    if (!G.act[q]) continue;
    const int r1 = (r0 + BM - 1 < p.n_q - 1) ? r0 + BM - 1 : p.n_q - 1;
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

__device__ __forceinline__ bool needs(const Geo& G, int q, int j) {
  return G.act[q] && j >= G.jlo[q] && j <= G.jhi[q];
}

// ---------------------------------------------------------------- producer

// Rolling-buffer rows of one key tile with cp.async (general W and chunk start):
// rows whose position is not held by the ring (or is negative) are zero-filled.
template <int D>
__device__ __forceinline__ void ring_tile_cpasync(const Params& p, const Geo& G, const uint16_t* ring,
                                                  uint8_t* dst, int kb, int lane) {
  const int seq = p.seq_ids ? p.seq_ids[G.b] : 0;
  const bool seq_ok = seq >= 0 && seq < p.max_seqs;
  if (!seq_ok && lane == 0) record_error(p.err, HSWA_ERR_DEVICE_BOUNDS);
  const int64_t row_base = seq_ok ? (((int64_t)seq * p.n_swa + p.ring_layer) * p.Hkv + G.g) * p.window : 0;
  const int held_lo = (G.P - p.window > 0) ? G.P - p.window : 0;
  if (p.fp8) {
    const bool is_v = ring == p.ring_v;
    ring_rows_fp8<D>((is_v ? p.ring_v8 : p.ring_k8) + row_base * D, seq_ok, held_lo, G.P, p.window,
                     is_v ? p.v_scale[G.g] : p.k_scale[G.g], dst, kb, lane);
  } else {
    ring_rows_cpasync<D>(ring + row_base * D, seq_ok, held_lo, G.P, p.window, dst, kb, lane);
  }
}

// FP8 page tiles (full layers of an FP8 pool, head_dim 128): the producer loads a tile's 128 rows x
// 128 codes by TMA (128-byte swizzle) into the upper half of its bf16 stage buffer, which holds the
// tile's dims 64..127 afterwards; warps 10 and 11 turn it into bf16 in place, row by row (a thread
// owns whole rows: a row's codes and its upper bf16 half occupy the same 128 bytes, and the thread
// reads them before it writes). Values are code value times the KV head's scale, rounded to bf16.
// Rows past the last key of the unit are written as zeros. Then the buffer is handed to the MMA
// (k_full / v_full, one arrival per converting thread).
template <int D>
__device__ void page_converter(const Params& p, uint8_t* smem, Bars* bars) {
  using L = Layout<D>;
  static_assert(D == 128, "FP8 page tiles are converted for head_dim 128");
  const int ct = threadIdx.x - 10 * 32;  // 0 .. 63
  int it = 0;
  for (int rnd = 0, unit = cta_unit(0); unit < p.n_units; unit = cta_unit(++rnd)) {
    Geo G;
    make_geo(p, unit, G);
    int kmax = 0;
    for (int q = 0; q < NQT; ++q)
      if (G.act[q] && G.i1[q] > kmax) kmax = G.i1[q];
    for (int j = G.jb; j <= G.je; ++j, ++it) {
      const int s = it % NSTAGE;
      const uint32_t ph = (it / NSTAGE) & 1;
      const int kb = key_base(p, G, j);
      for (int kv = 0; kv < 2; ++kv) {
        if (!mbar_wait(kv ? &bars->raw_v[s] : &bars->raw_k[s], ph, p.err)) return;
        uint8_t* tile = smem + (kv ? L::V_OFF : L::K_OFF) + s * L::TILE;
        const float sc = kv ? p.v_scale[G.g] : p.k_scale[G.g];
#pragma unroll 1
        for (int rr = 0; rr < 2; ++rr) {
          const int r = ct + 64 * rr;
          const bool zero = kb + r > kmax;
          const int sw = r & 7;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            // codes of dims 64 half .. 64 half + 63: 16-byte chunks 4 half .. 4 half + 3 of row r
            uint4 x[4];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
              x[c4] = zero ? make_uint4(0, 0, 0, 0)
                           : *reinterpret_cast<const uint4*>(tile + L::BLOCK + r * 128 + (((4 * half + c4) ^ sw) << 4));
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const uint32_t w[4] = {x[c4].x, x[c4].y, x[c4].z, x[c4].w};
              uint32_t o[8];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                o[2 * i] = e4m3x2_scaled_bf16x2(w[i], sc);
                o[2 * i + 1] = e4m3x2_scaled_bf16x2(w[i] >> 16, sc);
              }
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int ch = 2 * c4 + h;  // bf16 chunk of block `half`
                *reinterpret_cast<uint4*>(tile + half * L::BLOCK + r * 128 + ((ch ^ sw) << 4)) =
                    make_uint4(o[4 * h], o[4 * h + 1], o[4 * h + 2], o[4 * h + 3]);
              }
            }
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(kv ? &bars->v_full[s] : &bars->k_full[s]);
      }
    }
  }
}

template <int D>
__device__ void producer(const Params& p, uint8_t* smem, Bars* bars, const CUtensorMap* tm_q,
                         const CUtensorMap* tm_k, const CUtensorMap* tm_v, const CUtensorMap* tm_rk,
                         const CUtensorMap* tm_rv) {
  using L = Layout<D>;
  const int lane = threadIdx.x & 31;
  int it = 0;        // K/V tiles loaded so far (stage ring position)
  uint32_t uq = 0;   // units started (Q buffer phase)
  uint32_t nfix = 0; // page tiles zero-filled past the last key (v_fix phase)
  for (int rnd = 0, unit = cta_unit(0); unit < p.n_units; unit = cta_unit(++rnd), ++uq) {
    Geo G;
    make_geo(p, unit, G);
    // the Q buffers are free once every S MMA of the previous unit has completed
    if (!mbar_wait(&bars->q_empty, (uq & 1) ^ 1, p.err)) return;
    if (lane == 0) {
      int nact = 0;
      for (int q = 0; q < NQT; ++q) nact += G.act[q];
      mbar_arrive_expect_tx(&bars->q_full, nact * L::TILE);
      for (int q = 0; q < NQT; ++q) {
        if (!G.act[q]) continue;
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_4d(smem + L::Q_OFF + q * L::TILE + dh * L::BLOCK, tm_q, &bars->q_full, dh * 64, G.hq[q],
                      G.t[q] * BM, G.b);
      }
    }
    __syncwarp();
    // highest key position any query of this unit may need
    int kmax = 0;
    for (int q = 0; q < NQT; ++q)
      if (G.act[q] && G.i1[q] > kmax) kmax = G.i1[q];
    const int seq = (!p.is_full && p.seq_ids) ? p.seq_ids[G.b] : 0;
    const bool ring_fast = p.ring_tma && (G.P % BN) == 0;

    for (int j = G.jb; j <= G.je; ++j, ++it) {
      const int s = it % NSTAGE;
      const uint32_t ph = (it / NSTAGE) & 1;
      const int kb = key_base(p, G, j);
      for (int kv = 0; kv < 2; ++kv) {
        uint64_t* full = kv ? &bars->v_full[s] : &bars->k_full[s];
        uint64_t* empty = kv ? &bars->v_empty[s] : &bars->k_empty[s];
        uint8_t* dst = smem + (kv ? L::V_OFF : L::K_OFF) + s * L::TILE;
        if (!mbar_wait(empty, ph ^ 1, p.err)) return;
        if (p.is_full && p.conv) {
          // FP8 pages: the codes go to the upper half of the stage buffer; page_converter makes bf16
          uint64_t* raw = kv ? &bars->raw_v[s] : &bars->raw_k[s];
          if (lane == 0) {
            mbar_arrive_expect_tx(raw, BN * D);
            const CUtensorMap* tm = kv ? tm_v : tm_k;
            for (int half = 0; half < 2; ++half) {
              const int pos0 = kb + 64 * half;
              const int lp = pos0 / 64;
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
              tma_load_3d(dst + L::BLOCK + half * 64 * 128, tm, raw, 0, 0, (int)row);
            }
          }
        } else if (p.is_full) {
          // Rows of the last page past the last key hold stale memory; P is 0 there, but
          // 0 * NaN would still poison P V, so that V tile is zeroed past kmax before use.
          const bool fix = kv == 1 && kb <= kmax && kmax < kb + BN - 1 && ((kmax + 1) % 64) != 0;
          uint64_t* land = fix ? &bars->v_fix : full;
          if (lane == 0) {
            mbar_arrive_expect_tx(land, L::TILE);
            const CUtensorMap* tm = kv ? tm_v : tm_k;
            for (int half = 0; half < 2; ++half) {
              const int pos0 = kb + 64 * half;
              const int lp = pos0 / 64;
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
            if (!mbar_wait(&bars->v_fix, nfix & 1, p.err)) return;
            ++nfix;
            const int r0 = (int)(kmax - kb + 1);
            for (int idx = lane; idx < (BN - r0) * (D / 8); idx += 32) {
              const int r = r0 + idx / (D / 8);
              const int c = idx % (D / 8);
              *reinterpret_cast<uint4*>(dst + (c >> 3) * L::BLOCK + r * 128 + (c & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
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
}

// ---------------------------------------------------------------- MMA issuer

template <int D>
__device__ void mma_issuer(const Params& p, uint8_t* smem, Bars* bars, uint32_t tbase) {
  using L = Layout<D>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
  const uint32_t q_base = smem_u32(smem + L::Q_OFF);
  const uint32_t k_base = smem_u32(smem + L::K_OFF);
  const uint32_t v_base = smem_u32(smem + L::V_OFF);

  uint32_t np[NQT] = {0, 0};  // P tiles consumed per query tile (p_full phase)
  int it = 0;                 // K/V tiles consumed (stage ring position)
  uint32_t uq = 0;
  for (int rnd = 0, unit = cta_unit(0); unit < p.n_units; unit = cta_unit(++rnd), ++uq) {
    Geo G;
    make_geo(p, unit, G);
    if (!mbar_wait(&bars->q_full, uq & 1, p.err)) return;
    tc_fence_after();

    bool pend[NQT] = {false, false};
    bool started[NQT] = {false, false};
    int prev_s = 0;
    uint32_t prev_ph = 0;
    bool have_prev = false;

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
    auto drain_q = [&](int q, bool& v_ready) -> bool {
      if (!mbar_wait(&bars->p_full[q], np[q] & 1, p.err)) return false;
      ++np[q];
      tc_fence_after();
      if (!v_ready) {
        if (!mbar_wait(&bars->v_full[prev_s], prev_ph, p.err)) return false;
        tc_fence_after();
        v_ready = true;
      }
      issue_pv(q, prev_s);
      pend[q] = false;
      return true;
    };

    for (int j = G.jb; j <= G.je; ++j, ++it) {
      const int s = it % NSTAGE;
      const uint32_t ph = (it / NSTAGE) & 1;
      if (!mbar_wait(&bars->k_full[s], ph, p.err)) return;
      tc_fence_after();
      bool v_ready = false;
      for (int q = 0; q < NQT; ++q) {
        if (pend[q] && !drain_q(q, v_ready)) return;
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
      if (have_prev) {
        if (!v_ready) {
          if (!mbar_wait(&bars->v_full[prev_s], prev_ph, p.err)) return;
          tc_fence_after();
        }
        umma_commit(&bars->v_empty[prev_s]);
      }
      prev_s = s;
      prev_ph = ph;
      have_prev = true;
    }
    // every S MMA of the unit is issued: the Q buffers can be refilled once they complete
    umma_commit(&bars->q_empty);
    // drain the last tile's P V products and release its V stage
    bool v_ready = false;
    for (int q = 0; q < NQT; ++q)
      if (pend[q] && !drain_q(q, v_ready)) return;
    if (have_prev) {
      if (!v_ready) {
        if (!mbar_wait(&bars->v_full[prev_s], prev_ph, p.err)) return;
        tc_fence_after();
      }
      umma_commit(&bars->v_empty[prev_s]);
    }
    for (int q = 0; q < NQT; ++q)
      if (G.act[q]) umma_commit(&bars->o_full[q]);
  }
}

// ---------------------------------------------------------------- softmax + epilogue

template <int D>
__device__ void softmax_wg(const Params& p, uint8_t* smem, Bars* bars, uint32_t tbase, const int q,
                           const CUtensorMap* tm_o) {
  using L = Layout<D>;
  const int wq = (threadIdx.x >> 5) & 3;
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;
  const uint32_t trow = tbase + ((uint32_t)(wq * 32) << 16);
  const uint32_t s_col = q * 128;
  const uint32_t o_col = L::O_COL0 + q * L::O_STRIDE;
  const float sl2 = p.scale_log2;
  uint32_t ns = 0;  // S tiles consumed (s_full phase)
  uint32_t no = 0;  // units finished (o_full phase)

  for (int rnd = 0, unit = cta_unit(0); unit < p.n_units; unit = cta_unit(++rnd)) {
    Geo G;
    make_geo(p, unit, G);
    // this warpgroup's query tile, as scalars (one code path for both warpgroups)
    const bool act = q ? G.act[1] : G.act[0];
    if (!act) continue;
    const int qi0 = q ? G.i0[1] : G.i0[0];
    const int qi1 = q ? G.i1[1] : G.i1[0];
    const int qjlo = q ? G.jlo[1] : G.jlo[0];
    const int qjhi = q ? G.jhi[1] : G.jhi[0];
    const int qt = q ? G.t[1] : G.t[0];
    const int lo_last = window_lo(p, qi1);
    const int i = qi0 + r;
    const int lo_i = window_lo(p, i);
    float m_used = -INFINITY;
    float l = 0.f;
    uint32_t n_done = 0;

    for (int j = qjlo; j <= qjhi; ++j) {
      if (!mbar_wait(&bars->s_full[q], ns & 1, p.err)) return;
      ++ns;
      tc_fence_after();
      // columns of this row inside the band: [c_lo, c_hi] (edge tiles only)
      const int kb = key_base(p, G, j);
      const bool edge = !(kb + BN - 1 <= qi0 && kb >= lo_last);
      const int c_lo = lo_i - kb;
      const int c_hi = i - kb;
      softmax_tile<D, 1>(trow, s_col, o_col, sl2, edge, c_lo, c_hi, m_used, l, n_done > 0);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[q]);
      ++n_done;
    }

    if (!mbar_wait(&bars->o_full[q], no & 1, p.err)) return;
    ++no;
    tc_fence_after();
    store_output<D>(trow, o_col, l, smem + L::O_OFF + q * L::BLOCK + wq * 4096, lane, tm_o, q ? G.hq[1] : G.hq[0],
                    qt * BM + wq * 32, G.b, p.n_q);
    // O of this query tile has been read: the next unit's first P V may overwrite it
    // (ordered by this warpgroup's next p_full arrival).
    tc_fence_before();
  }
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_rk, const __grid_constant__ CUtensorMap tm_rv,
                   const __grid_constant__ CUtensorMap tm_o) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::BAR_OFF);
  const int warp = threadIdx.x >> 5;

  if (read_error(p.err) != 0) return;  // a pending device error: skip the work

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&bars->k_full[s], p.conv ? 64 : 1);  // converting threads, or the loading thread
      mbar_init(&bars->v_full[s], p.conv ? 64 : 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->raw_k[s], 1);
      mbar_init(&bars->raw_v[s], 1);
    }
    for (int q = 0; q < NQT; ++q) {
      mbar_init(&bars->s_full[q], 1);
      mbar_init(&bars->p_full[q], 128);
      mbar_init(&bars->o_full[q], 1);
    }
    mbar_init(&bars->v_fix, 1);
    fence_barrier_init();
  }
  if (warp == PRODUCER_WARP && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_o);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
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
    // two softmax warpgroups take the registers the third one gives back
    asm volatile("setmaxnreg.inc.sync.aligned.u32 " HSWA_STR(HSWA_SOFTMAX_REGS) ";" ::: "memory");
    softmax_wg<D>(p, smem, bars, tbase, warp >> 2, &tm_o);
    if ((threadIdx.x & 31) == 0) bulk_wait_all();  // output stores complete before the CTA exits
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 " HSWA_STR(HSWA_PRODUCER_REGS) ";" ::: "memory");
    if (warp == PRODUCER_WARP) {
      producer<D>(p, smem, bars, &tm_q, &tm_k, &tm_v, &tm_rk, &tm_rv);
    } else if (warp == MMA_WARP) {
      if ((threadIdx.x & 31) == 0) mma_issuer<D>(p, smem, bars, tbase);
      __syncwarp();
    } else if (p.conv) {
      if constexpr (D == 128) page_converter<D>(p, smem, bars);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace

int launch_prefill(const PrefillLaunch& Lc, cudaStream_t stream) {
  // narrow windows: every query tile's band fits in two key tiles, which stay resident while
  // all query heads of a KV head pass through them
  if (Lc.window >= 1 && Lc.window <= BN + 1) return launch_prefill_narrow(Lc, stream);
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
  p.ring_k = pool->ring_k;
  p.ring_v = pool->ring_v;
  p.ring_k8 = pool->ring_k8;
  p.ring_v8 = pool->ring_v8;
  p.fp8 = pool->fp8 ? 1 : 0;
  p.conv = (pool->fp8 && Lc.window == 0) ? 1 : 0;
  if (pool->fp8) {
    const int n_layers = D.n_swa_layers + D.n_full_layers;
    p.k_scale = pool->scales + (size_t)(0 * n_layers + Lc.layer) * D.n_kv_heads;
    p.v_scale = pool->scales + (size_t)(1 * n_layers + Lc.layer) * D.n_kv_heads;
  }
  p.ring_layer = Lc.ring_layer;
  p.n_swa = D.n_swa_layers;
  p.max_seqs = D.max_seqs;
  p.ring_tma = pool->ring_tma ? 1 : 0;
  p.full_layer = Lc.full_layer;
  p.pages = D.pages_per_full_layer;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)Lc.d));
  p.n_pairs = (int)((Lc.n_q + BM * NQT - 1) / (BM * NQT));
  p.n_tiles = (int)((Lc.n_q + BM - 1) / BM);
  p.head_pairs = (p.G % 2) == 0 ? 1 : 0;
  {
    const int n_t = p.head_pairs ? p.n_tiles : p.n_pairs;
    p.t_block = HSWA_UNIT_TBLOCK > 0 && HSWA_UNIT_TBLOCK < n_t ? HSWA_UNIT_TBLOCK : (n_t > 0 ? n_t : 1);
  }
  p.max_start = 0x7fffffffLL - Lc.n_q - 2 * BN;
  p.err = pool->err;
  if (Lc.n_q == 0 || Lc.B == 0) return HSWA_OK;
  const int64_t units = p.head_pairs ? (int64_t)p.n_tiles * Lc.B * Lc.Hkv * (p.G / 2)
                                     : (int64_t)p.n_pairs * Lc.B * Lc.Hq;
  if (units > 0x7fffffff - 65536) {  // the unit index of every round stays below 2^31
    set_error("prefill: too many work units");
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  p.n_units = (int)units;
  const int sms = pool->sms;
  const int grid = p.n_units < sms ? p.n_units : sms;

  const CUtensorMap& rk = pool->ring_tma ? pool->tm_ring_k : Lc.tm_k;
  const CUtensorMap& rv = pool->ring_tma ? pool->tm_ring_v : Lc.tm_v;
  if (p.conv && Lc.d != 128) {
    set_error("prefill: FP8 pages are read with head_dim 128 only");
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  if (Lc.d == 128) {
    const int smem = Layout<128>::BYTES + 1024;
    cudaFuncSetAttribute(prefill_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_kernel<128><<<grid, NTHREADS, smem, stream>>>(p, Lc.tm_q, Lc.tm_k, Lc.tm_v, rk, rv, Lc.tm_o);
  } else {
    const int smem = Layout<64>::BYTES + 1024;
    cudaFuncSetAttribute(prefill_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_kernel<64><<<grid, NTHREADS, smem, stream>>>(p, Lc.tm_q, Lc.tm_k, Lc.tm_v, rk, rv, Lc.tm_o);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("prefill: launch failed: %s", cudaGetErrorString(e));
    return HSWA_ERR_CUDA;
  }
  return HSWA_OK;
}

}  // namespace hswa

// prefill_tile.cuh -- per-tile pieces shared by the prefill kernels: the online-softmax step of
// one 128-key tile for one query row (one thread per TMEM lane), the output epilogue, and the
// cp.async loader for rolling-buffer rows.
//
// Math ("Sliding Window Attention (SWA) no riron to jisso", section "formal definition",
// eqs. (1)-(5)): row i's weights are softmax_j(q_i . k_j / sqrt(d)) over the keys of its band;
// the step keeps the running maximum in the exp2 domain and rescales O only when the maximum
// grows by more than 2^kTau, so P = 2^(s * scale * log2 e - m) stays below 2^kTau.
#pragma once
#include "common.cuh"

namespace hswa {
namespace {

constexpr int BM = 128;     // query rows per tile
constexpr int BN = 128;     // keys per tile
constexpr float kTau = 8.0f;  // lazy rescale threshold (log2 units): P stays <= 2^8

// Tuning parameters (compile-time):
//  HSWA_POLY_PER8           pairs of scores in every 8 whose exponential runs on the FMA pipe
//  HSWA_SOFTMAX_SINGLE_PASS 1: keep all 128 scores of a row in registers (one TMEM read);
//                           0: read S twice (row maximum, then exponentials), fewer registers
//  HSWA_SOFTMAX_REGS / HSWA_PRODUCER_REGS  setmaxnreg split (2 * 128 * a + 128 * b <= 384 * 168)
//  HSWA_UNIT_TBLOCK         prefill unit order: query tiles per block (0: the whole chunk)
//  HSWA_UNIT_SERPENTINE     1: CTAs take the rounds of units in alternating directions
#ifndef HSWA_POLY_PER8
#define HSWA_POLY_PER8 0
#endif
#ifndef HSWA_SOFTMAX_SINGLE_PASS
#define HSWA_SOFTMAX_SINGLE_PASS 1
#endif
#ifndef HSWA_SOFTMAX_REGS
#define HSWA_SOFTMAX_REGS 208
#endif
#ifndef HSWA_PRODUCER_REGS
#define HSWA_PRODUCER_REGS 88
#endif
#ifndef HSWA_UNIT_TBLOCK
#define HSWA_UNIT_TBLOCK 1
#endif
#ifndef HSWA_UNIT_SERPENTINE
#define HSWA_UNIT_SERPENTINE 1
#endif
static_assert(2 * 128 * HSWA_SOFTMAX_REGS + 128 * HSWA_PRODUCER_REGS <= 384 * 168, "register split");
#define HSWA_STR2(x) #x
#define HSWA_STR(x) HSWA_STR2(x)

__device__ __forceinline__ constexpr bool use_poly(int pair) { return (pair & 7) >= 8 - HSWA_POLY_PER8; }

// One key tile of one query row. trow: this warp's TMEM lane base; S of the row in columns
// [s_col, s_col + 128), O in [o_col, o_col + D). Columns outside [c_lo, c_hi] are masked when
// `edge`. m_used / l: running maximum (log2 domain) and row sum; o_live: O already holds a
// partial sum (it is rescaled when the maximum moves). P is written over S as packed bf16;
// the caller waits for the TMEM stores and signals the MMA.
// MASK_MODE selects how edge tiles are masked (all give the same result):
//  0  per-column compares (faster where every tile is an edge tile, as in the narrow kernel);
//  1  integer sign arithmetic on every column (faster where edge tiles are few);
//  2  W = 128 with no row's band clipped at the sequence start (the narrow kernel's common tile):
//     before the diagonal a row keeps columns k > r, on the diagonal k <= r, so for warp w
//     (rows 32w .. 32w + 31) chunk w is the only chunk the band edge crosses and every other
//     chunk is wholly in or out for the whole warp. The warp loads chunk (w + c) & 3 into
//     register block c (rot = w), masks block 0 by lane and selects the other blocks whole;
//     `lower_edge` marks the tile before the diagonal. Single-pass softmax only.
template <int D, int MASK_MODE>
__device__ __forceinline__ void softmax_tile(uint32_t trow, uint32_t s_col, uint32_t o_col, float sl2, bool edge,
                                             int c_lo, int c_hi, float& m_used, float& l, bool o_live,
                                             int rot = 0, bool lower_edge = false) {
  static_assert(MASK_MODE != 2 || HSWA_SOFTMAX_SINGLE_PASS, "the rotated mask needs the single-pass softmax");
  constexpr bool BRANCH_FREE_MASK = MASK_MODE == 1;
  const int rc = MASK_MODE == 2 ? rot : 0;  // chunk rotation (0 folds away in the other modes)
#if HSWA_SOFTMAX_SINGLE_PASS
    // all 128 scores of the row: four TMEM loads, one wait
    uint32_t v[128];
    tmem_ld32_into<0>(trow + s_col + 32 * ((rc + 0) & 3), v);
    tmem_ld32_into<32>(trow + s_col + 32 * ((rc + 1) & 3), v);
    tmem_ld32_into<64>(trow + s_col + 32 * ((rc + 2) & 3), v);
    tmem_ld32_into<96>(trow + s_col + 32 * ((rc + 3) & 3), v);
    tmem_wait_ld();
    reg_fence_into<0>(v);
    reg_fence_into<32>(v);
    reg_fence_into<64>(v);
    reg_fence_into<96>(v);
    if (MASK_MODE == 2) {
      // block 0 = chunk rot: the lower edge keeps j > lane, the diagonal keeps j <= lane
      const int lane = threadIdx.x & 31;
      if (lower_edge) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j <= lane) v[j] = 0xFF800000u;
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j > lane) v[j] = 0xFF800000u;
      }
#pragma unroll
      for (int c = 1; c < 4; ++c) {
        // chunk rot + c lies above the warp's rows (kept before the diagonal, dropped on it);
        // a wrapped chunk lies below them
        const bool out = lower_edge ? (rc + c > 3) : (rc + c <= 3);
#pragma unroll
        for (int j = 32 * c; j < 32 * c + 32; ++j) v[j] = out ? 0xFF800000u : v[j];
      }
    } else if (edge) {
      if (BRANCH_FREE_MASK) {
        // the sign of (k - c_lo) | (c_hi - k) is set exactly outside [c_lo, c_hi] (positions
        // stay below 2^31 - 256, so neither difference overflows)
        const int nlo = -c_lo;
#pragma unroll
        for (int k = 0; k < 128; ++k) {
          const uint32_t m = (uint32_t)(((k + nlo) | (c_hi - k)) >> 31);
          v[k] = (v[k] & ~m) | (0xFF800000u & m);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 128; ++k)
          if (k < c_lo || k > c_hi) v[k] = __float_as_uint(-INFINITY);
      }
    }
    float m0 = __uint_as_float(v[0]), m1 = __uint_as_float(v[1]);
    float m2 = __uint_as_float(v[2]), m3 = __uint_as_float(v[3]);
#pragma unroll
    for (int k = 4; k < 124; k += 8) {
      m0 = fmax3(m0, __uint_as_float(v[k + 0]), __uint_as_float(v[k + 1]));
      m1 = fmax3(m1, __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
      m2 = fmax3(m2, __uint_as_float(v[k + 4]), __uint_as_float(v[k + 5]));
      m3 = fmax3(m3, __uint_as_float(v[k + 6]), __uint_as_float(v[k + 7]));
    }
    m0 = fmax3(m0, __uint_as_float(v[124]), __uint_as_float(v[125]));
    m1 = fmax3(m1, __uint_as_float(v[126]), __uint_as_float(v[127]));
    const float mx = fmaxf(fmax3(m0, m1, m2), m3);
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
    if (__any_sync(0xffffffffu, resc) && o_live) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(trow + o_col + c0, o);
        tmem_wait_ld();
        reg_fence32(o);
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
        tmem_st32(trow + o_col + c0, o);
      }
      tmem_wait_st();
    }
    // P = 2^(s * scale * log2 e - m) in place, packed to bf16 and stored over S
    const float moff = (m_used == -INFINITY) ? 0.f : m_used;
    const uint64_t scale2 = f2_pack(sl2, sl2);
    const uint64_t neg2 = f2_pack(-moff, -moff);
    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int c0 = 0; c0 < BN; c0 += 32) {
      uint32_t pk[16];
      if (MASK_MODE == 2 && c0 > 0) {
        // a block wholly outside every row's band: P = 0 without exponentials
        const bool out = lower_edge ? (rc + (c0 >> 5) > 3) : (rc + (c0 >> 5) <= 3);
        if (out) {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;
          tmem_st16(trow + s_col + 16 * (((c0 >> 5) + rc) & 3), pk);
          continue;
        }
      }
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        const int pair = (c0 + k) >> 1;
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(v[c0 + k]), __uint_as_float(v[c0 + k + 1])), scale2, neg2);
        uint64_t e;
        if (use_poly(pair)) {
          e = exp2_poly_x2(x);
        } else {
          float x0, x1;
          f2_unpack(x, x0, x1);
          e = f2_pack(ex2_approx(x0), ex2_approx(x1));
        }
        acc[pair & 3] = f2_add(acc[pair & 3], e);
        float e0, e1;
        f2_unpack(e, e0, e1);
        pk[k >> 1] = pack_bf16x2(e0, e1);
      }
      tmem_st16(trow + s_col + 16 * (((c0 >> 5) + rc) & 3), pk);
    }
#else
    // pass 1: row maximum, 64 scores at a time
    float mx = -INFINITY;
#pragma unroll
    for (int h2 = 0; h2 < BN; h2 += 64) {
      uint32_t va[32], vb[32];
      tmem_ld32(trow + s_col + h2, va);
      tmem_ld32(trow + s_col + h2 + 32, vb);
      tmem_wait_ld();
      reg_fence32(va);
      reg_fence32(vb);
      if (edge) {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const uint32_t ma = (uint32_t)(((h2 + k - c_lo) | (c_hi - h2 - k)) >> 31);
          const uint32_t mb = (uint32_t)(((h2 + 32 + k - c_lo) | (c_hi - h2 - 32 - k)) >> 31);
          va[k] = (va[k] & ~ma) | (0xFF800000u & ma);
          vb[k] = (vb[k] & ~mb) | (0xFF800000u & mb);
        }
      }
      float m0 = mx, m1 = __uint_as_float(va[0]), m2 = __uint_as_float(vb[0]);
#pragma unroll
      for (int k = 1; k < 31; k += 2) {
        m0 = fmax3(m0, __uint_as_float(va[k]), __uint_as_float(va[k + 1]));
        m1 = fmax3(m1, __uint_as_float(vb[k]), __uint_as_float(vb[k + 1]));
      }
      m2 = fmax3(m2, __uint_as_float(va[31]), __uint_as_float(vb[31]));
      mx = fmax3(m0, m1, m2);
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
    if (__any_sync(0xffffffffu, resc) && o_live) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(trow + o_col + c0, o);
        tmem_wait_ld();
        reg_fence32(o);
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
        tmem_st32(trow + o_col + c0, o);
      }
      tmem_wait_st();
    }
    // pass 2: P = 2^(s * scale * log2 e - m), 32 columns at a time, the next chunk's TMEM
    // load in flight while this one is exponentiated, packed and stored over S.
    const float moff = (m_used == -INFINITY) ? 0.f : m_used;
    const uint64_t scale2 = f2_pack(sl2, sl2);
    const uint64_t neg2 = f2_pack(-moff, -moff);
    uint64_t acc[4] = {0, 0, 0, 0};
    uint32_t buf[2][32];
    tmem_ld32(trow + s_col, buf[0]);
    tmem_wait_ld();
    reg_fence32(buf[0]);
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t(&cur)[32] = buf[c & 1];
      if (c + 1 < BN / 32) tmem_ld32(trow + s_col + 32 * (c + 1), buf[(c + 1) & 1]);
      const int c0 = 32 * c;
      if (edge) {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const uint32_t m = (uint32_t)(((c0 + k - c_lo) | (c_hi - c0 - k)) >> 31);
          cur[k] = (cur[k] & ~m) | (0xFF800000u & m);
        }
      }
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        const int pair = (c0 + k) >> 1;
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(cur[k]), __uint_as_float(cur[k + 1])), scale2, neg2);
        uint64_t e;
        if (use_poly(pair)) {
          e = exp2_poly_x2(x);
        } else {
          float x0, x1;
          f2_unpack(x, x0, x1);
          e = f2_pack(ex2_approx(x0), ex2_approx(x1));
        }
        acc[pair & 3] = f2_add(acc[pair & 3], e);
        float e0, e1;
        f2_unpack(e, e0, e1);
        pk[k >> 1] = pack_bf16x2(e0, e1);
      }
      tmem_st16(trow + s_col + (c0 >> 1), pk);
      if (c + 1 < BN / 32) {
        tmem_wait_ld();
        reg_fence32(buf[(c + 1) & 1]);
      }
    }
#endif
    float a0, a1, b0, b1, c0_, c1_, d0, d1;
    f2_unpack(acc[0], a0, a1);
    f2_unpack(acc[1], b0, b1);
    f2_unpack(acc[2], c0_, c1_);
    f2_unpack(acc[3], d0, d1);
    l += ((a0 + a1) + (b0 + b1)) + ((c0_ + c1_) + (d0 + d1));
}

// Epilogue of one query tile: O / l -> bf16, staged per warp (its 32 rows x 128 B, 128-byte
// swizzle, 4 KB at `stage`) and written by one TMA store per 64-column half into the output
// map at (column, head h, row0 .. row0 + 31, batch b); rows past n_q fall outside the map.
template <int D>
__device__ __forceinline__ void store_output(uint32_t trow, uint32_t o_col, float l, uint8_t* stage, int lane,
                                             const CUtensorMap* tm_o, int h, int row0, int b, int n_q) {
  const float inv = 1.f / l;
#pragma unroll
  for (int dh = 0; dh < D / 64; ++dh) {
    if (lane == 0) bulk_wait_read_all();  // the previous store from this buffer has read it
    __syncwarp();
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(trow + o_col + dh * 64 + c0, o);
      tmem_wait_ld();
      reg_fence32(o);
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 32; k += 2)
        pk[k >> 1] = pack_bf16x2(__uint_as_float(o[k]) * inv, __uint_as_float(o[k + 1]) * inv);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int chunk = (c0 >> 3) + x;
        *reinterpret_cast<uint4*>(stage + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
            make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && row0 < n_q) {  // a box wholly past the chunk end is not issued
      tma_store_4d(tm_o, stage, dh * 64, h, row0, b);
      bulk_commit_group();
    }
  }
}

// store_output for a caller whose next MMA waits for O's TMEM columns: all D columns of the row
// are read into registers first, `o_free` gets this thread's arrival (the columns may be
// overwritten from then on), and the packing, staging and TMA stores follow.
template <int D>
__device__ __forceinline__ void store_output_release(uint32_t trow, uint32_t o_col, float l, uint8_t* stage, int lane,
                                                     const CUtensorMap* tm_o, int h, int row0, int b, int n_q,
                                                     uint64_t* o_free) {
  uint32_t o[D];
  tmem_ld32_into<0>(trow + o_col, o);
  tmem_ld32_into<32>(trow + o_col + 32, o);
  if constexpr (D == 128) {
    tmem_ld32_into<64>(trow + o_col + 64, o);
    tmem_ld32_into<96>(trow + o_col + 96, o);
  }
  tmem_wait_ld();
  reg_fence_into<0>(o);
  reg_fence_into<32>(o);
  if constexpr (D == 128) {
    reg_fence_into<64>(o);
    reg_fence_into<96>(o);
  }
  tc_fence_before();
  mbar_arrive(o_free);
  const float inv = 1.f / l;
#pragma unroll
  for (int dh = 0; dh < D / 64; ++dh) {
    if (lane == 0) bulk_wait_read_all();  // the previous store from this buffer has read it
    __syncwarp();
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 32) {
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 32; k += 2)
        pk[k >> 1] = pack_bf16x2(__uint_as_float(o[dh * 64 + c0 + k]) * inv,
                                 __uint_as_float(o[dh * 64 + c0 + k + 1]) * inv);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int chunk = (c0 >> 3) + x;
        *reinterpret_cast<uint4*>(stage + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
            make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && row0 < n_q) {  // a box wholly past the chunk end is not issued
      tma_store_4d(tm_o, stage, dh * 64, h, row0, b);
      bulk_commit_group();
    }
  }
}

// Rolling-buffer rows of one key tile with cp.async (any W and chunk start), one warp:
// positions kb .. kb + 127 come from slot pos mod W of the ring at `ring_rows` (W rows of d),
// rows whose position the ring does not hold ([held_lo, held_hi) holds) or a bad ring are
// zero-filled. Layout of dst: [D / 64 blocks][128 rows][128 B], 128-byte swizzle, consecutive
// 64-dim blocks blk_stride bytes apart (16 KB for one tile; a tile inside a taller operand
// leaves room for the other rows).
template <int D>
__device__ __forceinline__ void ring_rows_cpasync(const uint16_t* ring_rows, bool ok, int held_lo, int held_hi,
                                                  int W, uint8_t* dst, int kb, int lane, int blk_stride = BM * 128) {
  const uint32_t sdst = smem_u32(dst);
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int idx = lane; idx < BN * CH; idx += 32) {
    const int r = idx / CH;
    const int c = idx % CH;
    const int pos = kb + r;
    const bool held = ok && pos >= held_lo && pos < held_hi;
    const uint16_t* src = held ? ring_rows + (int64_t)(pos % W) * D + c * 8 : ring_rows;
    const int blk = c >> 3, cc = c & 7;
    const uint32_t off = blk * blk_stride + r * 128 + ((cc ^ (r & 7)) << 4);
    cp_async_16(sdst + off, src, held ? 16u : 0u);
  }
  cp_async_wait_all();
  fence_proxy_async_smem();
  __syncwarp();
}

// Two E4M3 codes (the low 16 bits of x) -> their fp32 values times `scale`, packed to bf16x2
// (the E4M3 -> f16 step is exact; the product rounds once to fp32 and once to bf16).
__device__ __forceinline__ uint32_t e4m3x2_scaled_bf16x2(uint32_t x, float scale) {
  uint32_t h;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "r"(x));
  float lo, hi;
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
  return pack_bf16x2(lo * scale, hi * scale);
}

// ring_rows_cpasync for a ring of FP8 E4M3 codes: the held rows are dequantized (code value times
// `scale`) to bf16 in the tile's swizzled layout; the others are zero. One warp, plain loads
// (four 16-byte loads in flight per lane); the caller fences and signals as for the cp.async path.
template <int D>
__device__ __forceinline__ void ring_rows_fp8(const uint8_t* ring_rows, bool ok, int held_lo, int held_hi, int W,
                                              float scale, uint8_t* dst, int kb, int lane, int blk_stride = BM * 128) {
  constexpr int CH8 = D / 16;           // 16-code chunks per row
  constexpr int TOTAL = BN * CH8;       // chunks per tile
  constexpr int BATCH = 4;
  static_assert(TOTAL % (32 * BATCH) == 0, "tile chunks");
  for (int base = 0; base < TOTAL; base += 32 * BATCH) {
    uint4 x[BATCH];
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      const int idx = base + u * 32 + lane;
      const int r = idx / CH8, c = idx % CH8;
      const int pos = kb + r;
      const bool held = ok && pos >= held_lo && pos < held_hi;
      x[u] = held ? __ldg(reinterpret_cast<const uint4*>(ring_rows + (int64_t)(pos % W) * D + c * 16))
                  : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      const int idx = base + u * 32 + lane;
      const int r = idx / CH8, c = idx % CH8;
      const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
      uint32_t o[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[2 * i] = e4m3x2_scaled_bf16x2(w[i], scale);
        o[2 * i + 1] = e4m3x2_scaled_bf16x2(w[i] >> 16, scale);
      }
      // codes 16c .. 16c + 15 -> bf16 chunks 2c and 2c + 1 of the row
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int cc = 2 * c + h;
        const int blk = cc >> 3, ch = cc & 7;
        *reinterpret_cast<uint4*>(dst + blk * blk_stride + r * 128 + ((ch ^ (r & 7)) << 4)) =
            make_uint4(o[4 * h], o[4 * h + 1], o[4 * h + 2], o[4 * h + 3]);
      }
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
}

}  // namespace
}  // namespace hswa

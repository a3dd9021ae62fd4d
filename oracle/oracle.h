/*
 * oracle.h -- plain, slow, obviously correct fp64 CPU reference for hybrid
 * sliding-window attention and its dual-pool KV cache.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this code. It shares no
 * code with the CUDA library (no headers, no helpers, no tables) and never
 * reads a ring buffer or a page table: keys and values are indexed by their
 * logical position.
 *
 * Sources (the pages these functions restate):
 *  - "Sliding Window Attention (SWA) no riron to jisso" (disassemble-channel.com),
 *    section "formal definition": eq.(1) the window W(i) = {j : max(0,i-w+1) <= j <= i},
 *    eq.(2) the 0/1 mask, eq.(3) masked scaled scores q.k/sqrt(d_k) or -inf,
 *    eq.(4) softmax over the row, eq.(5) o_i = sum_j alpha_ij v_j.
 *  - same page, section "Mistral: SWA and GQA": several query heads share one
 *    KV head (32 query heads : 8 KV heads); KV bytes = 2 * n * h * d_k * sizeof.
 *  - same page, section "Rolling Buffer KV Cache": slot idx(t) = t mod w, eq.(7).
 *  - "MiMo v2.5 inference optimisation" (youngju.dev), section "KV cache
 *    redesign": dual pool, window-safe length (the tail W tokens of a prefix
 *    match must have valid SWA slots); section "architecture": 60 SWA + 10 full
 *    layers, KV ratio (60 W + 10 N) / (70 N).
 *
 * Readings taken where the pages are silent or garbled:
 *  - positions are 0-based (eq.(1) uses max(0, .)); eq.(4)'s k = 1..n is read as
 *    the same 0-based row;
 *  - GQA maps query head h to KV head floor(h / (Hq / Hkv));
 *  - scale is 1/sqrt(head_dim); no bias, softcap or RoPE (RoPE is taken as
 *    already applied to q and k);
 *  - window 0 stands for full causal attention (the W >= N case);
 *  - window_safe_len checks the literal tail of W positions [L-W, L-1].
 */
#ifndef HSWA_ORACLE_H
#define HSWA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Number of (i, j) pairs with j in W(i), 0 <= i < n  (window 0 = full causal). */
int64_t orc_mask_count(int64_t n, int64_t window);

/* Attention rows over a logical key/value sequence.
 *  q      [n_rows][n_q_heads][head_dim]  bf16 bit patterns
 *  q_pos  [n_rows]                       absolute position i of each query row
 *  k, v   [n_keys][n_kv_heads][head_dim] bf16 bit patterns; row r holds position key_base + r
 *  window >= 1 for sliding-window attention, 0 for full causal attention
 *  out    [n_rows][n_q_heads][head_dim]  fp64
 * Returns 0, or -1 when a needed key position is not inside [key_base, key_base + n_keys)
 * or the head counts are inconsistent. */
int orc_attention(const uint16_t* q, const int64_t* q_pos, int64_t n_rows, int n_q_heads,
                  const uint16_t* k, const uint16_t* v, int64_t key_base, int64_t n_keys,
                  int n_kv_heads, int head_dim, int64_t window, double* out, int n_threads);

/* orc_attention with fp64 keys and values ([n_keys][n_kv_heads][head_dim]), e.g. entries of an
 * FP8 KV cache dequantized with orc_e4m3_decode times their scale, mixed with bf16 ones. */
int orc_attention_kv64(const uint16_t* q, const int64_t* q_pos, int64_t n_rows, int n_q_heads,
                       const double* k, const double* v, int64_t key_base, int64_t n_keys,
                       int n_kv_heads, int head_dim, int64_t window, double* out, int n_threads);

/* FP8 E4M3 (OCP 8-bit floating point formats specification: 1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, no infinities, S.1111.111 = NaN, largest finite magnitude 448) -- the storage
 * format of an FP8 KV cache ("MiMo v2.5 inference optimisation", closing section: quantization
 * cuts the bits per cached entry and stacks with the sliding window's cut in entries).
 * decode: the value of a code. encode: round to nearest, ties to even, saturating at +-448.
 * quantize: out[i] = encode(fp32(bf16 x[i]) * (1.0f / scale)) with both operations in fp32. */
double orc_e4m3_decode(uint8_t code);
uint8_t orc_e4m3_encode(double x);
int orc_e4m3_quantize(const uint16_t* x, int64_t n, float scale, uint8_t* out);

/* Window-safe prefix-match length, by definition.
 * For request r: match length m, cached length C, and a W-bit slot-valid mask
 * (valid[r * ((W + 31) / 32) + s / 32] bit s % 32 for ring slot s).
 * resident(p) <=> max(0, C - W) <= p < C  and  valid[p mod W]
 * safe(L)     <=> every p in [max(0, L - W), L - 1] is resident   (safe(0) holds)
 * out[r]       = max { L in [0, m] : safe(L) }.
 * Returns 0, or -1 on bad arguments (W < 1, negative m or C). */
int orc_window_safe_len(const int64_t* m, const int64_t* cached, const uint32_t* valid,
                        int32_t window, int64_t n_req, int64_t* out);

/* Rolling buffer after appending positions 0 .. n_appended-1 one by one into a
 * w-slot ring with slot = pos mod w: slot_pos[s] = position held by slot s, or -1. */
int orc_ring_trace(int64_t n_appended, int64_t w, int64_t* slot_pos);

/* KV bytes of `layers` layers holding `tokens` token-slots each:
 * 2 (K and V) * layers * kv_heads * tokens * head_dim * elem_bytes. */
int64_t orc_kv_bytes(int64_t layers, int64_t kv_heads, int64_t tokens, int64_t head_dim,
                     int64_t elem_bytes);

/* Dual-pool ratio of hybrid KV to all-full KV: (n_swa W + n_full N) / ((n_swa + n_full) N). */
double orc_hybrid_kv_ratio(int64_t n_swa, int64_t n_full, int64_t window, int64_t n_tokens);

#ifdef __cplusplus
}
#endif
#endif

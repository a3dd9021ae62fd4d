// shard.cpp -- how the hot path splits over several GPUs (host code).
//
// Prefill: by KV head. Attention of query head h reads only KV head h / G ("Sliding Window
// Attention (SWA) no riron to jisso", section "Mistral: SWA and GQA"), so a rank that owns KV
// heads [g0, g1) and query heads [g0 G, g1 G) holds that slice of every pool and computes its
// outputs with no exchange; the outputs are gathered only when a caller needs them replicated.
// Decode: by sequence, every sequence on one rank, the ranks' total context balanced greedily with
// the longest sequences placed first in length buckets ("MiMo v2.5 inference optimisation",
// section "KV cache redesign": length buckets 0-64K / 64K-256K / 256K-1M keep batches even).
#include <algorithm>
#include <cstdint>
#include <numeric>
#include <vector>

#include "../../include/hswa.h"

namespace hswa {
void set_error(const char* fmt, ...);
}

extern "C" {

int hswa_shard_kv_heads(int32_t n_kv_heads, int32_t n_ranks, int32_t rank, int32_t* head_begin,
                        int32_t* head_end) {
  if (n_kv_heads < 1 || n_ranks < 1 || rank < 0 || rank >= n_ranks || !head_begin || !head_end) {
    hswa::set_error("hswa_shard_kv_heads: bad arguments");
    return HSWA_ERR_INVALID_ARG;
  }
  if (n_kv_heads % n_ranks != 0) {
    hswa::set_error("hswa_shard_kv_heads: %d KV heads do not split evenly over %d ranks", n_kv_heads, n_ranks);
    return HSWA_ERR_UNSUPPORTED_SHAPE;
  }
  const int32_t per = n_kv_heads / n_ranks;
  *head_begin = rank * per;
  *head_end = rank * per + per;
  return HSWA_OK;
}

int hswa_shard_sequences(const int64_t* ctx_len, int32_t n_seqs, int32_t n_ranks, int32_t* rank_of_seq,
                         int64_t* load_per_rank) {
  if (n_seqs < 0 || n_ranks < 1 || (n_seqs > 0 && (!ctx_len || !rank_of_seq))) {
    hswa::set_error("hswa_shard_sequences: bad arguments");
    return HSWA_ERR_INVALID_ARG;
  }
  for (int32_t s = 0; s < n_seqs; ++s)
    if (ctx_len[s] < 0) {
      hswa::set_error("hswa_shard_sequences: negative context length");
      return HSWA_ERR_INVALID_ARG;
    }
  auto bucket = [](int64_t L) { return L >= 262144 ? 2 : (L >= 65536 ? 1 : 0); };
  std::vector<int32_t> order(n_seqs);
  std::iota(order.begin(), order.end(), 0);
  // longest bucket first, longest first inside a bucket, then by index (a deterministic order)
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
    const int ba = bucket(ctx_len[a]), bb = bucket(ctx_len[b]);
    if (ba != bb) return ba > bb;
    return ctx_len[a] > ctx_len[b];
  });
  std::vector<int64_t> load(n_ranks, 0);
  for (int32_t s : order) {
    int32_t best = 0;
    for (int32_t r = 1; r < n_ranks; ++r)
      if (load[r] < load[best]) best = r;  // least loaded, lowest rank on ties
    rank_of_seq[s] = best;
    load[best] += ctx_len[s];
  }
  if (load_per_rank)
    for (int32_t r = 0; r < n_ranks; ++r) load_per_rank[r] = load[r];
  return HSWA_OK;
}

}  // extern "C"

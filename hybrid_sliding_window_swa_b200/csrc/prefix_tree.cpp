// prefix_tree.cpp -- SWA-aware prefix cache over a token trie (host code).
//
// "MiMo v2.5 inference optimisation", section "KV cache redesign" (SWA-aware prefix cache):
// a prefix cache reuses KV on the premise that equal token sequences give equal KV, but with
// sliding-window layers only the tail of a cached sequence's window KV survives (or none of it),
// so a match is cut to the window-safe length: the tail W positions must still hold valid
// sliding-window KV. This file keeps that state per position of a token trie: every cached
// position keeps its full-attention KV (pages), while a position's sliding-window KV is held only
// while some cached sequence's window covers it (the last W positions of that sequence) and it
// has not been evicted. A match walks the trie and returns the common-prefix length m and the
// largest L <= m whose tail [max(0, L - W), L) is held, so a request can resume at L.
//
// With one cached sequence of length C this reduces to window_safe_len (a ring of W slots holding
// positions [max(0, C - W), C)); here eviction is per position and cached sequences share prefixes.
#include <cstdint>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/hswa.h"

namespace hswa {
void set_error(const char* fmt, ...);
}

struct hswa_prefix_tree {
  int32_t window;
  // node 0 is the root (no token); node k > 0 is one position: depth[k] = position + 1
  std::vector<int32_t> parent;
  std::vector<int32_t> token;
  std::vector<int64_t> depth;
  std::vector<uint32_t> swa_refs;  // cached sequences whose window covers this position (0 after eviction)
  std::unordered_map<uint64_t, int32_t> child;  // (parent, token) -> node

  static uint64_t key(int32_t p, int32_t t) { return ((uint64_t)(uint32_t)p << 32) | (uint32_t)t; }
  int32_t find(int32_t p, int32_t t) const {
    auto it = child.find(key(p, t));
    return it == child.end() ? -1 : it->second;
  }
};

namespace {

bool check_tokens(const int32_t* tokens, int64_t n, const char* who) {
  if (n < 0 || (n > 0 && !tokens)) {
    hswa::set_error("%s: bad token array", who);
    return false;
  }
  return true;
}

}  // namespace

extern "C" {

int hswa_tree_create(int32_t window, hswa_prefix_tree** out) {
  if (!out || window < 1) {
    hswa::set_error("hswa_tree_create: window must be >= 1 and out non-null");
    return HSWA_ERR_INVALID_ARG;
  }
  hswa_prefix_tree* t = new (std::nothrow) hswa_prefix_tree();
  if (!t) {
    hswa::set_error("hswa_tree_create: out of host memory");
    return HSWA_ERR_OUT_OF_MEMORY;
  }
  t->window = window;
  t->parent.push_back(-1);
  t->token.push_back(0);
  t->depth.push_back(0);
  t->swa_refs.push_back(0);
  *out = t;
  return HSWA_OK;
}

int hswa_tree_destroy(hswa_prefix_tree* t) {
  delete t;
  return HSWA_OK;
}

int hswa_tree_insert(hswa_prefix_tree* t, const int32_t* tokens, int64_t n, int64_t* new_nodes) {
  if (!t) {
    hswa::set_error("hswa_tree_insert: null tree");
    return HSWA_ERR_INVALID_ARG;
  }
  if (!check_tokens(tokens, n, "hswa_tree_insert")) return HSWA_ERR_INVALID_ARG;
  if ((int64_t)t->parent.size() + n > INT32_MAX) {
    hswa::set_error("hswa_tree_insert: tree would exceed 2^31 nodes");
    return HSWA_ERR_OUT_OF_MEMORY;
  }
  int64_t added = 0;
  int32_t node = 0;
  const int64_t win_lo = n > t->window ? n - t->window : 0;
  try {
    for (int64_t p = 0; p < n; ++p) {
      int32_t c = t->find(node, tokens[p]);
      if (c < 0) {
        c = (int32_t)t->parent.size();
        t->parent.push_back(node);
        t->token.push_back(tokens[p]);
        t->depth.push_back(p + 1);
        t->swa_refs.push_back(0);
        t->child.emplace(hswa_prefix_tree::key(node, tokens[p]), c);
        ++added;
      }
      if (p >= win_lo) ++t->swa_refs[c];  // this sequence's window: its last W positions
      node = c;
    }
  } catch (const std::bad_alloc&) {
    hswa::set_error("hswa_tree_insert: out of host memory");
    return HSWA_ERR_OUT_OF_MEMORY;
  }
  if (new_nodes) *new_nodes = added;
  return HSWA_OK;
}

int hswa_tree_release(hswa_prefix_tree* t, const int32_t* tokens, int64_t n) {
  if (!t) {
    hswa::set_error("hswa_tree_release: null tree");
    return HSWA_ERR_INVALID_ARG;
  }
  if (!check_tokens(tokens, n, "hswa_tree_release")) return HSWA_ERR_INVALID_ARG;
  const int64_t win_lo = n > t->window ? n - t->window : 0;
  int32_t node = 0;
  for (int64_t p = 0; p < n; ++p) {
    node = t->find(node, tokens[p]);
    if (node < 0) {
      hswa::set_error("hswa_tree_release: sequence is not cached");
      return HSWA_ERR_INVALID_ARG;
    }
    if (p >= win_lo && t->swa_refs[node] > 0) --t->swa_refs[node];
  }
  return HSWA_OK;
}

int hswa_tree_evict_swa(hswa_prefix_tree* t, const int32_t* tokens, int64_t n, int64_t pos_lo, int64_t pos_hi,
                        int64_t* evicted) {
  if (!t) {
    hswa::set_error("hswa_tree_evict_swa: null tree");
    return HSWA_ERR_INVALID_ARG;
  }
  if (!check_tokens(tokens, n, "hswa_tree_evict_swa")) return HSWA_ERR_INVALID_ARG;
  int64_t count = 0;
  int32_t node = 0;
  for (int64_t p = 0; p < n && p < pos_hi; ++p) {
    node = t->find(node, tokens[p]);
    if (node < 0) break;  // positions past the cached part hold nothing to evict
    if (p >= pos_lo && t->swa_refs[node] > 0) {
      t->swa_refs[node] = 0;
      ++count;
    }
  }
  if (evicted) *evicted = count;
  return HSWA_OK;
}

int hswa_tree_match(const hswa_prefix_tree* t, const int32_t* tokens, int64_t n, int64_t* match_len,
                    int64_t* safe_len) {
  if (!t || !match_len || !safe_len) {
    hswa::set_error("hswa_tree_match: null argument");
    return HSWA_ERR_INVALID_ARG;
  }
  if (!check_tokens(tokens, n, "hswa_tree_match")) return HSWA_ERR_INVALID_ARG;
  // walk the common prefix; run = consecutive held positions ending at p
  const int64_t W = t->window;
  int32_t node = 0;
  int64_t m = 0, run = 0, best = 0;
  for (int64_t p = 0; p < n; ++p) {
    node = t->find(node, tokens[p]);
    if (node < 0) break;
    m = p + 1;
    run = t->swa_refs[node] > 0 ? run + 1 : 0;
    // L = p + 1 is safe when its tail [max(0, L - W), L) is held
    if (run >= (m < W ? m : W)) best = m;
  }
  *match_len = m;
  *safe_len = best;
  return HSWA_OK;
}

int hswa_tree_match_batch(const hswa_prefix_tree* t, const int32_t* tokens, const int64_t* offsets, int32_t n_req,
                          int64_t* match_len, int64_t* safe_len) {
  if (!t || !offsets || !match_len || !safe_len || n_req < 0) {
    hswa::set_error("hswa_tree_match_batch: bad arguments");
    return HSWA_ERR_INVALID_ARG;
  }
  for (int32_t r = 0; r < n_req; ++r) {
    const int64_t a = offsets[r], b = offsets[r + 1];
    if (a < 0 || b < a) {
      hswa::set_error("hswa_tree_match_batch: offsets must be non-decreasing from 0");
      return HSWA_ERR_INVALID_ARG;
    }
    const int rc = hswa_tree_match(t, tokens + a, b - a, match_len + r, safe_len + r);
    if (rc) return rc;
  }
  return HSWA_OK;
}

int hswa_tree_stats(const hswa_prefix_tree* t, int64_t* n_positions, int64_t* n_swa_held) {
  if (!t) {
    hswa::set_error("hswa_tree_stats: null tree");
    return HSWA_ERR_INVALID_ARG;
  }
  int64_t held = 0;
  for (size_t k = 1; k < t->swa_refs.size(); ++k) held += t->swa_refs[k] > 0;
  if (n_positions) *n_positions = (int64_t)t->parent.size() - 1;
  if (n_swa_held) *n_swa_held = held;
  return HSWA_OK;
}

}  // extern "C"

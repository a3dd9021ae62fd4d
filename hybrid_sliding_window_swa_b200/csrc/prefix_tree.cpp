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
//
// Every insert names an owner: the ring row where the caller keeps that sequence's sliding-window
// KV. A position's holders are the owners whose window covers it and whose copy has not been
// evicted since they were inserted; it holds sliding-window KV while it has a holder. A match can
// report, for each ring slot of the resumed window, one holder's ring row, which is where that
// position's KV can be copied from (slot = position mod W in every ring).
#include <algorithm>
#include <cstdint>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/hswa.h"

namespace hswa {
void set_error(const char* fmt, ...);
}

struct hswa_prefix_tree {
  // Path-compressed trie: node k holds a run of consecutive cached positions (its label) and,
  // per position, the number of holders (owners whose window covers it and whose copy was not
  // evicted since). Node 0 is the root with an empty label. A child is found by (node, first
  // token). Each cached position has a stable id (pid0 + offset in the label; a split keeps the
  // ids) that keys its holders and the owners of the inserts ending there.
  struct Node {
    int64_t pos0;                 // position of the label's first token
    int64_t pid0;                 // id of the label's first position
    std::vector<int32_t> label;   // tokens at positions pos0 .. pos0 + label.size() - 1
    std::vector<uint32_t> refs;   // per position of the label: number of holders
    std::vector<int32_t> kids;    // children (their first tokens key the lookup map)
  };
  int32_t window;
  std::vector<Node> nodes;
  std::unordered_map<uint64_t, int32_t> child;  // (node, first token of the child's label) -> child
  std::unordered_map<int64_t, std::vector<int32_t>> holders;     // position id -> owners (refs > 0 only)
  std::unordered_map<int64_t, std::vector<int32_t>> end_owners;  // position id -> owners of inserts ending there
  int64_t n_positions = 0;
  int64_t next_pid = 0;

  static uint64_t key(int32_t n, int32_t t) { return ((uint64_t)(uint32_t)n << 32) | (uint32_t)t; }
  int32_t find(int32_t n, int32_t t) const {
    auto it = child.find(key(n, t));
    return it == child.end() ? -1 : it->second;
  }

  // Visit the cached positions along tokens[0..n) in order, as runs inside node labels:
  // f(node, offset in label, position, run length). Stops where the path leaves the tree;
  // returns the number of positions visited (the common-prefix length).
  template <class F>
  int64_t walk(const int32_t* tokens, int64_t n, F&& f) const {
    int32_t node = 0;
    size_t off = 0;  // offset inside the current node's label; the root's label is empty
    int64_t i = 0;
    while (i < n) {
      const Node* nd = &nodes[node];
      if (off == nd->label.size()) {
        const int32_t c = find(node, tokens[i]);
        if (c < 0) break;
        node = c;
        off = 0;
        nd = &nodes[node];
      }
      // longest run of equal tokens inside this label
      const size_t lim = std::min<size_t>(nd->label.size() - off, (size_t)(n - i));
      size_t k = 0;
      while (k < lim && nd->label[off + k] == tokens[i + k]) ++k;
      if (k == 0) break;
      f(node, off, i, (int64_t)k);
      off += k;
      i += (int64_t)k;
      if (off < nd->label.size()) break;  // diverged (or ran out of tokens) inside the label
    }
    return i;
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
  t->nodes.push_back(hswa_prefix_tree::Node{0, 0, {}, {}, {}});
  *out = t;
  return HSWA_OK;
}

int hswa_tree_destroy(hswa_prefix_tree* t) {
  delete t;
  return HSWA_OK;
}

int hswa_tree_insert(hswa_prefix_tree* t, const int32_t* tokens, int64_t n, int32_t owner, int64_t* new_nodes) {
  if (!t) {
    hswa::set_error("hswa_tree_insert: null tree");
    return HSWA_ERR_INVALID_ARG;
  }
  if (!check_tokens(tokens, n, "hswa_tree_insert")) return HSWA_ERR_INVALID_ARG;
  int64_t added = 0;
  try {
    // 1. structure: follow the cached prefix, split the label where the path leaves it, and
    //    attach the rest of the sequence as one new node
    int32_t node = 0;
    size_t off = 0;
    int64_t i = 0;
    while (i < n) {
      hswa_prefix_tree::Node* nd = &t->nodes[node];
      if (off == nd->label.size()) {
        const int32_t c = t->find(node, tokens[i]);
        if (c < 0) break;
        node = c;
        off = 0;
        continue;
      }
      if (nd->label[off] != tokens[i]) {
        // split node at off: the head keeps [0, off), a new tail node takes the rest and the
        // old children
        if (t->nodes.size() >= (size_t)INT32_MAX - 2) {
          hswa::set_error("hswa_tree_insert: tree would exceed 2^31 nodes");
          return HSWA_ERR_OUT_OF_MEMORY;
        }
        const int32_t tail = (int32_t)t->nodes.size();
        hswa_prefix_tree::Node tn;
        tn.pos0 = nd->pos0 + (int64_t)off;
        tn.pid0 = nd->pid0 + (int64_t)off;
        tn.label.assign(nd->label.begin() + off, nd->label.end());
        tn.refs.assign(nd->refs.begin() + off, nd->refs.end());
        t->nodes.push_back(std::move(tn));
        nd = &t->nodes[node];  // the vector may have moved
        // the old children now hang under the tail node
        t->nodes[tail].kids.swap(nd->kids);
        for (int32_t c : t->nodes[tail].kids) {
          const int32_t tok = t->nodes[c].label[0];
          t->child.erase(hswa_prefix_tree::key(node, tok));
          t->child[hswa_prefix_tree::key(tail, tok)] = c;
        }
        nd->kids.assign(1, tail);
        t->child[hswa_prefix_tree::key(node, t->nodes[tail].label[0])] = tail;
        nd->label.resize(off);
        nd->refs.resize(off);
        break;
      }
      ++off;
      ++i;
    }
    if (i < n) {
      if (t->nodes.size() >= (size_t)INT32_MAX - 2) {
        hswa::set_error("hswa_tree_insert: tree would exceed 2^31 nodes");
        return HSWA_ERR_OUT_OF_MEMORY;
      }
      const int32_t fresh = (int32_t)t->nodes.size();
      hswa_prefix_tree::Node fn;
      fn.pos0 = i;
      fn.pid0 = t->next_pid;
      fn.label.assign(tokens + i, tokens + n);
      fn.refs.assign((size_t)(n - i), 0u);
      t->nodes.push_back(std::move(fn));
      t->next_pid += n - i;
      t->nodes[node].kids.push_back(fresh);
      t->child[hswa_prefix_tree::key(node, tokens[i])] = fresh;
      added = n - i;
      t->n_positions += added;
    }
  } catch (const std::bad_alloc&) {
    hswa::set_error("hswa_tree_insert: out of host memory");
    return HSWA_ERR_OUT_OF_MEMORY;
  }
  // 2. this sequence's window, its last W positions, gains the owner as a holder, and one more
  //    insert by this owner ends at its last position
  const int64_t win_lo = n > t->window ? n - t->window : 0;
  try {
    t->walk(tokens, n, [&](int32_t node, size_t off, int64_t pos, int64_t len) {
      hswa_prefix_tree::Node& nd = t->nodes[node];
      for (int64_t k = 0; k < len; ++k) {
        const int64_t pid = nd.pid0 + (int64_t)off + k;
        if (pos + k >= win_lo) {
          t->holders[pid].push_back(owner);
          ++nd.refs[off + (size_t)k];
        }
        if (pos + k == n - 1) t->end_owners[pid].push_back(owner);
      }
    });
  } catch (const std::bad_alloc&) {
    hswa::set_error("hswa_tree_insert: out of host memory");
    return HSWA_ERR_OUT_OF_MEMORY;
  }
  if (new_nodes) *new_nodes = added;
  return HSWA_OK;
}

int hswa_tree_release(hswa_prefix_tree* t, const int32_t* tokens, int64_t n, int32_t owner) {
  if (!t) {
    hswa::set_error("hswa_tree_release: null tree");
    return HSWA_ERR_INVALID_ARG;
  }
  if (!check_tokens(tokens, n, "hswa_tree_release")) return HSWA_ERR_INVALID_ARG;
  if (n == 0) return HSWA_OK;  // the empty sequence holds nothing
  // the sequence must be cached with an insert of exactly these tokens by this owner left
  int64_t end_pid = -1;
  const int64_t m = t->walk(tokens, n, [&](int32_t node, size_t off, int64_t pos, int64_t len) {
    if (pos + len == n) end_pid = t->nodes[node].pid0 + (int64_t)off + len - 1;
  });
  auto eo = m == n ? t->end_owners.find(end_pid) : t->end_owners.end();
  auto hit = eo == t->end_owners.end() ? std::vector<int32_t>::iterator()
                                       : std::find(eo->second.begin(), eo->second.end(), owner);
  if (eo == t->end_owners.end() || hit == eo->second.end()) {
    hswa::set_error("hswa_tree_release: no insert of exactly this sequence by owner %d is left to release", owner);
    return HSWA_ERR_INVALID_ARG;
  }
  eo->second.erase(hit);
  if (eo->second.empty()) t->end_owners.erase(eo);
  // the owner stops holding its window (positions evicted since its insert no longer list it)
  const int64_t win_lo = n > t->window ? n - t->window : 0;
  t->walk(tokens, n, [&](int32_t node, size_t off, int64_t pos, int64_t len) {
    hswa_prefix_tree::Node& nd = t->nodes[node];
    for (int64_t k = 0; k < len; ++k) {
      if (pos + k < win_lo) continue;
      auto h = t->holders.find(nd.pid0 + (int64_t)off + k);
      if (h == t->holders.end()) continue;
      auto o = std::find(h->second.begin(), h->second.end(), owner);
      if (o == h->second.end()) continue;
      h->second.erase(o);
      nd.refs[off + (size_t)k] = (uint32_t)h->second.size();
      if (h->second.empty()) t->holders.erase(h);
    }
  });
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
  t->walk(tokens, n < pos_hi ? n : (pos_hi > 0 ? pos_hi : 0), [&](int32_t node, size_t off, int64_t pos, int64_t len) {
    hswa_prefix_tree::Node& nd = t->nodes[node];
    for (int64_t k = 0; k < len; ++k) {
      uint32_t& r = nd.refs[off + (size_t)k];
      if (pos + k >= pos_lo && r > 0) {
        r = 0;
        t->holders.erase(nd.pid0 + (int64_t)off + k);
        ++count;
      }
    }
  });
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
  const int64_t W = t->window;
  int64_t run = 0, best = 0;  // run: consecutive positions holding sliding-window KV
  const int64_t m = t->walk(tokens, n, [&](int32_t node, size_t off, int64_t pos, int64_t len) {
    const uint32_t* r = t->nodes[node].refs.data() + off;
    for (int64_t k = 0; k < len; ++k) {
      run = r[k] > 0 ? run + 1 : 0;
      const int64_t L = pos + k + 1;  // safe when its tail [max(0, L - W), L) is held
      if (run >= (L < W ? L : W)) best = L;
    }
  });
  *match_len = m;
  *safe_len = best;
  return HSWA_OK;
}

int hswa_tree_match_slots(const hswa_prefix_tree* t, const int32_t* tokens, int64_t n, int64_t* match_len,
                          int64_t* safe_len, int32_t* slot_owner) {
  if (!slot_owner) {
    hswa::set_error("hswa_tree_match_slots: null slot_owner");
    return HSWA_ERR_INVALID_ARG;
  }
  const int rc = hswa_tree_match(t, tokens, n, match_len, safe_len);
  if (rc) return rc;
  const int64_t W = t->window, L = *safe_len;
  for (int64_t s = 0; s < W; ++s) slot_owner[s] = -1;
  const int64_t lo = L > W ? L - W : 0;
  t->walk(tokens, L, [&](int32_t node, size_t off, int64_t pos, int64_t len) {
    for (int64_t k = 0; k < len; ++k) {
      if (pos + k < lo) continue;
      auto h = t->holders.find(t->nodes[node].pid0 + (int64_t)off + k);
      // every position of the safe tail has a holder; the most recent insert is reported
      if (h != t->holders.end() && !h->second.empty()) slot_owner[(pos + k) % W] = h->second.back();
    }
  });
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
  for (const auto& nd : t->nodes)
    for (uint32_t r : nd.refs) held += r > 0;
  if (n_positions) *n_positions = t->n_positions;
  if (n_swa_held) *n_swa_held = held;
  return HSWA_OK;
}

}  // extern "C"
